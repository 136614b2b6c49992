"""Benchmark of the fused-convolution hot path on B200.

One step = one pass of both fused operations over their full-size synthetic
workloads, inputs resident in device memory:

  op A  conv2d x[128,8,384,384] (Cout 64, 3x3, stride 1, no pad) -> AvgPool2d(4)
        -> sigmoid -> sum -> out[128]
  op B  depthwise(K 9, stride 1, pad 4) + pointwise(256 -> 512) conv1d
        x[32,256,4096] -> out[32,512,4096]

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fcv|reference]
Under torchrun each rank runs its own replica of the step (the batch items are
independent; there is no data-path collective) and rank 0 prints one JSON line
with the whole-job throughput.  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead (rank 0 only).
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from direct_convolution_chip_b200 import workloads as wl  # noqa: E402

METRIC = "fused-conv GFLOP/s (2·MACs/s) and % of B200 roofline per config"
UNIT = "GFLOP/s"
SPEC_FMA_LANES_PER_SM = 128       # FP32 FMA units per SM
SPEC_SM_MAX_MHZ = 1965.0          # clocks.max.sm
TF32_OVER_BF16 = 1.1 / 2.25       # nominal dense TF32 : BF16 tensor throughput
ALGO_NAMES = {10: "conv2d_direct_fma", 11: "conv2d_poolfirst_fma", 12: "conv2d_tc_3xtf32",
              13: "conv2d_tc_shift_3xtf32",
              20: "dwsep_conv1d_fma", 21: "dwsep_conv1d_tc_register_halo", 22: "dwsep_conv1d_tc_2sm",
              23: "dwsep_conv1d_tc_tma_halo"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

CASE_A = wl.CONV2D_FULL
CASE_B = wl.CONV1D_FULL


# ----------------------------------------------------------------------------
# work accounting (algorithmic MACs and compulsory bytes)
# ----------------------------------------------------------------------------

def macs_conv2d(N, Cin, H, W, Cout, P):
    """MACs of the direct method: every conv output inside a pooled window, 9*Cin each."""
    PH, PW = (H - 2) // P, (W - 2) // P
    return N * Cout * (PH * P) * (PW * P) * Cin * 9


def bytes_conv2d(N, Cin, H, W, Cout, P):
    return 4 * (N * Cin * H * W + Cout * Cin * 9 + Cout + N)


def macs_conv1d(N, C, T, O, K, s, p):
    To = (T + 2 * p - K) // s + 1
    return N * C * To * K + N * O * C * To


def macs_conv1d_pointwise(N, C, T, O, K, s, p):
    To = (T + 2 * p - K) // s + 1
    return N * O * C * To


def bytes_conv1d(N, C, T, O, K, s, p, bias=True):
    To = (T + 2 * p - K) // s + 1
    return 4 * (N * C * T + C * K + O * C + (O if bias else 0) + N * O * To)


def case_macs(c):
    if c.op == "conv2d":
        return macs_conv2d(c.N, c.Cin, c.H, c.W, c.Cout, c.P)
    return macs_conv1d(c.N, c.C, c.T, c.O, c.K, c.stride, c.pad)


def case_bytes(c):
    if c.op == "conv2d":
        return bytes_conv2d(c.N, c.Cin, c.H, c.W, c.Cout, c.P)
    return bytes_conv1d(c.N, c.C, c.T, c.O, c.K, c.stride, c.pad, c.has_bias)


def workload_name():
    a, b = CASE_A, CASE_B
    return (f"conv2d x[{a.N},{a.Cin},{a.H},{a.W}] Cout {a.Cout} 3x3 -> AvgPool2d({a.P}) -> sigmoid -> sum "
            f"+ dwsep conv1d x[{b.N},{b.C},{b.T}] K {b.K} s {b.stride} p {b.pad} -> [{b.N},{b.O},{b.T}]")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def fma_peak_tflops(props):
    """FP32 FMA roofline from unit counts and the maximum SM clock."""
    return props.multi_processor_count * SPEC_FMA_LANES_PER_SM * 2 * SPEC_SM_MAX_MHZ * 1e6 / 1e12


def roofline_time_s(macs, nbytes, peak_tflops, hbm_gbs):
    return max(2.0 * macs / (peak_tflops * 1e12), nbytes / (hbm_gbs * 1e9))


def op_roofline(c, tensor, tc_peak, fma_peak, hbm):
    """Roofline time of one workload.  FP32-FMA kernels: every MAC on the FMA
    pipe.  Tensor-core kernels: conv2d's MACs on the 3xTF32 tensor pipe;
    conv1d's pointwise MACs on the tensor pipe while its depthwise MACs run
    on the FMA pipe beside them.  Then the slower of that and the compulsory
    bytes at HBM bandwidth."""
    nbytes = case_bytes(c)
    t_mem = nbytes / (hbm * 1e9)
    if not tensor:
        return max(2.0 * case_macs(c) / (fma_peak * 1e12), t_mem)
    if c.op == "conv2d":
        return max(2.0 * case_macs(c) / (tc_peak * 1e12), t_mem)
    pw = macs_conv1d_pointwise(c.N, c.C, c.T, c.O, c.K, c.stride, c.pad)
    dw = case_macs(c) - pw
    return max(2.0 * pw / (tc_peak * 1e12), 2.0 * dw / (fma_peak * 1e12), t_mem)


def stats_ms(values):
    """Median, min and 90th percentile of a list of times (ms)."""
    v = sorted(values)
    return {"median": v[len(v) // 2], "min": v[0], "p90": v[min(len(v) - 1, int(0.9 * len(v)))], "n": len(v)}


def source_info():
    """Git commit when the checkout has one, and a hash of the library and bench sources."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "direct_convolution_chip_b200", "csrc")
    files = sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    for f in files + [os.path.join(ROOT, "include", "fcv.h"), os.path.abspath(__file__)]:
        with open(f, "rb") as fh:
            h.update(fh.read())
    try:
        sha = subprocess.run(["git", "-C", ROOT, "rev-parse", "HEAD"], capture_output=True, text=True,
                             timeout=10).stdout.strip() or None
    except (OSError, subprocess.SubprocessError):
        sha = None
    return {"git_sha": sha, "source_sha256": h.hexdigest()}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def probe_tf32_tflops():
    """Dense TF32 tensor rate measured now on this GPU: one CTA per SM issuing
    tcgen05.mma kind::tf32 M = 128, N = 256, K = 8 back to back (best of 3)."""
    import ctypes
    from direct_convolution_chip_b200 import build as fcv_build
    try:
        lib = ctypes.CDLL(fcv_build.build_probes())
    except (OSError, subprocess.SubprocessError):
        return None
    best = None
    for _ in range(3):
        f, ms, cyc = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
        if lib.fcvprobe_tf32_mma_rate(256, 0, 1, 1, 24000, ctypes.byref(f), ctypes.byref(ms), ctypes.byref(cyc)) == 0:
            best = max(best or 0.0, f.value / 1e12)
    return best


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    """SM clock, power and clock-event reasons sampled while the timed region
    runs: NVML every ~2 ms in a thread (nvidia-smi every 100 ms when NVML is
    not importable); mark() brackets the samples that count."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    NVML_REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
                    0x4: "sw_power_cap"}

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.samples = []  # (time, sm_mhz, max_mhz, power_w, reason bits) from NVML
        self.stop_flag = False
        self.window = None
        self.nvml = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            handle = pynvml.nvmlDeviceGetHandleByUUID(sel.encode() if isinstance(sel, str) else sel)
            self.nvml = (pynvml, handle)
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", sel], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, RuntimeError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _poll_nvml(self):
        nv, h = self.nvml
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.perf_counter(), sm, mx, pw, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark(self, t0, t1):
        """Host-time window that contains the timed region."""
        self.window = (t0, t1)

    def stop(self):
        if self.nvml is not None:
            self.stop_flag = True
            if self.thread:
                self.thread.join(timeout=5)
            return self.summary_nvml()
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        return self.summary()

    def summary_nvml(self):
        rows = self.samples
        if self.window:
            inside = [r for r in rows if self.window[0] <= r[0] <= self.window[1]]
            rows = inside or rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "nvml"}
        reasons = sorted({name for r in rows for bit, name in self.NVML_REASONS.items() if r[4] & bit})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max(r[2] for r in rows),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r[3] for r in rows),
                "source": "nvml, every ~2 ms during the timed region"}

    def summary(self):
        sm, mx, pw = [], [], []
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                pw.append(float(parts[3]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(pw)}


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local, backend="nccl"):
    if world <= 1:
        return False
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=120)}
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, **kw)
    return True


def max_over_ranks(values, use_dist, device):
    """Element-wise max of a list of floats over all ranks."""
    if not use_dist:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(use_dist, device=None):
    if use_dist:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------

def traffic_per_launch(kernel_key):
    """DRAM bytes per launch from the committed ncu capture, or None if the
    kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kernel_key)
    if not e:
        return None
    # "source" is one file or a list of files: the sha256 of their contents,
    # concatenated in order
    srcs = e["source"] if isinstance(e["source"], list) else [e["source"]]
    h = hashlib.sha256()
    try:
        for src in srcs:
            h.update(open(os.path.join(ROOT, src), "rb").read())
    except OSError:
        return None
    return e["bytes_per_launch"] if h.hexdigest() == e["source_sha256"] else None


def job_throughput(flops_per_rank_step, world, max_step_s):
    """Whole-job GFLOP/s: every rank's work divided by the slowest rank's step time."""
    return flops_per_rank_step * world / max_step_s / 1e9


def run_oracle_sample(budget_s=12.0):
    """Time the CPU oracle (as it stands) on whole batch items of both workloads,
    repeating full passes until about `budget_s` seconds of CPU work."""
    import oracle
    xa, wa, ba = wl.conv2d_inputs(CASE_A)
    xb, dwb, pwb, bb = wl.conv1d_inputs(CASE_B)
    xa, wa, ba = xa.numpy(), wa.numpy(), ba.numpy()
    xb, dwb, pwb, bb = xb.numpy(), dwb.numpy(), pwb.numpy(), bb.numpy()
    per_a = macs_conv2d(1, CASE_A.Cin, CASE_A.H, CASE_A.W, CASE_A.Cout, CASE_A.P)
    per_b = macs_conv1d(1, CASE_B.C, CASE_B.T, CASE_B.O, CASE_B.K, CASE_B.stride, CASE_B.pad)
    items_a = items_b = 0
    ta = tb = 0.0
    while ta + tb < budget_s:
        t = time.perf_counter()
        oracle.conv2d_pool_sigmoid_sum(xa, wa, ba, CASE_A.P)
        ta += time.perf_counter() - t
        items_a += CASE_A.N
        t = time.perf_counter()
        oracle.dwsep_conv1d(xb, dwb, pwb, bb, CASE_B.stride, CASE_B.pad)
        tb += time.perf_counter() - t
        items_b += CASE_B.N
    flops = 2.0 * (items_a * per_a + items_b * per_b)
    return {"value": flops / (ta + tb) / 1e9, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{items_a // CASE_A.N} full pass(es) of both workloads: op A {items_a} batch items "
                      f"({ta:.2f} s), op B {items_b} batch items ({tb:.2f} s); double-precision OpenMP loops"}


def time_small_case(lib, fcv, c, stream, flush_buf, iters=60):
    """Device time of one named small workload through its C entry point: warm
    L2 (inputs resident) and cold L2 (a 256 MB buffer written between calls),
    each over `iters` timed calls with CUDA events on the launching stream."""
    import ctypes
    P = ctypes.c_void_p
    sp = P(stream.cuda_stream)
    if c.op == "conv2d":
        x, w, b = [t.cuda() for t in wl.conv2d_inputs(c)]
        out = torch.empty((c.N,), device="cuda")

        def fn():
            return lib.fcv_conv2d_pool_sigmoid_sum(P(x.data_ptr()), P(w.data_ptr()), P(b.data_ptr()), c.N, c.Cin,
                                                   c.H, c.W, c.Cout, c.P, P(out.data_ptr()), sp)
        algo = fcv.conv2d_auto_algo(c.N, c.Cin, c.H, c.W, c.Cout, c.P)
    else:
        x, dw, pw, b = [t.cuda() for t in wl.conv1d_inputs(c)]
        To = (c.T + 2 * c.pad - c.K) // c.stride + 1
        out = torch.empty((c.N, c.O, To), device="cuda")

        def fn():
            return lib.fcv_dwsep_conv1d(P(x.data_ptr()), P(dw.data_ptr()), P(pw.data_ptr()), P(b.data_ptr()),
                                        c.N, c.C, c.T, c.O, c.K, c.stride, c.pad, P(out.data_ptr()), sp)
        algo = fcv.dwsep_conv1d_auto_algo(x, dw, pw, c.stride, c.pad)
    for _ in range(5):
        if fn() != 0:
            raise RuntimeError(f"{c.name}: launch failed")
    res = {}
    for leg in ("warm_l2", "cold_l2"):
        ts = []
        for _ in range(iters):
            if leg == "cold_l2":
                flush_buf.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        res[leg] = stats_ms(ts)
    return algo, res


def run_gpu(args):
    import direct_convolution_chip_b200 as fcv

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    use_dist = init_dist(world, local)
    lib = fcv.load()
    props = torch.cuda.get_device_properties(device)
    tf32_probe = probe_tf32_tflops() if world == 1 else None

    # Inputs: seeded synthetic data of the pages' shapes, resident in HBM.
    xa, wa, ba = wl.conv2d_inputs(CASE_A)
    xb, dwb, pwb, bb = wl.conv1d_inputs(CASE_B)
    host = [t.pin_memory() for t in (xa, wa, ba, xb, dwb, pwb, bb)]
    xa_d, wa_d, ba_d, xb_d, dwb_d, pwb_d, bb_d = [t.to(device) for t in host]
    out_a = torch.empty((CASE_A.N,), device=device)
    To = (CASE_B.T + 2 * CASE_B.pad - CASE_B.K) // CASE_B.stride + 1
    out_b = torch.empty((CASE_B.N, CASE_B.O, To), device=device)
    stream = torch.cuda.current_stream(device)
    sp = stream.cuda_stream

    import ctypes
    P = ctypes.c_void_p

    def op_a():
        st = lib.fcv_conv2d_pool_sigmoid_sum(P(xa_d.data_ptr()), P(wa_d.data_ptr()), P(ba_d.data_ptr()),
                                             CASE_A.N, CASE_A.Cin, CASE_A.H, CASE_A.W, CASE_A.Cout, CASE_A.P,
                                             P(out_a.data_ptr()), P(sp))
        if st:
            raise fcv.FcvError(st, "fcv_conv2d_pool_sigmoid_sum")

    def op_b():
        st = lib.fcv_dwsep_conv1d(P(xb_d.data_ptr()), P(dwb_d.data_ptr()), P(pwb_d.data_ptr()),
                                  P(bb_d.data_ptr()), CASE_B.N, CASE_B.C, CASE_B.T, CASE_B.O, CASE_B.K,
                                  CASE_B.stride, CASE_B.pad, P(out_b.data_ptr()), P(sp))
        if st:
            raise fcv.FcvError(st, "fcv_dwsep_conv1d")

    for _ in range(args.warmup):
        op_a()
        op_b()
    torch.cuda.synchronize(device)

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(use_dist, device)
    torch.cuda.synchronize(device)
    sampler.start()
    time.sleep(0.2)  # let the sampler attach before the timed region
    h0 = time.perf_counter()
    t_start.record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        op_a()
        ev[i][1].record(stream)
        op_b()
        ev[i][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark(h0, time.perf_counter())
    clocks = sampler.stop()
    barrier(use_dist, device)
    total_ms = t_start.elapsed_time(t_end)
    la = [e[0].elapsed_time(e[1]) for e in ev]
    lb = [e[1].elapsed_time(e[2]) for e in ev]
    ta_ms, tb_ms = sum(la), sum(lb)
    total_ms, ta_ms, tb_ms = max_over_ranks([total_ms, ta_ms, tb_ms], use_dist, device)

    # End to end through the public API with pinned host buffers: every step
    # copies its inputs host -> device, runs both ops and copies both results
    # back.  Each op of a step runs on its own stream, and steps alternate
    # between two such pairs (four streams); the binding does not wait for its
    # copies (wait=False).  So no input upload queues behind the other op's
    # kernel on the copy engine, one step's results travel device -> host
    # while the next step's inputs travel host -> device, and the timed region
    # ends when the last copy has landed.
    # 16 to 32 steps: the first step's uploads and the last step's compute and
    # downloads overlap nothing, and over few steps that fill and drain would
    # weigh on the per-step figure
    e2e_steps = max(16, min(32, K // 4))
    xa_h, wa_h, ba_h, xb_h, dwb_h, pwb_h, bb_h = host
    streams = [stream] + [torch.cuda.Stream(device) for _ in range(3)]  # (op A, op B) x 2 step parities
    ra_h = [torch.empty((CASE_A.N,), dtype=torch.float32, pin_memory=True) for _ in range(2)]
    rb_h = [torch.empty((CASE_B.N, CASE_B.O, To), dtype=torch.float32, pin_memory=True) for _ in range(2)]

    def e2e_step(i):
        sa, sb = streams[2 * (i & 1)], streams[2 * (i & 1) + 1]
        fcv.conv2d_pool_sigmoid_sum(xa_h, wa_h, ba_h, CASE_A.P, out=ra_h[i & 1], stream=sa, wait=False)
        fcv.dwsep_conv1d(xb_h, dwb_h, pwb_h, bb_h, CASE_B.stride, CASE_B.pad, out=rb_h[i & 1], stream=sb,
                         wait=False)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(device)
    barrier(use_dist, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(streams[0])
    for s_ in streams[1:]:
        s_.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    for s_ in streams[1:]:
        done = torch.cuda.Event()
        done.record(s_)
        streams[0].wait_event(done)
    e1.record(streams[0])
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], use_dist, device)[0]
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = ra_h[0].numel() * 4 + rb_h[0].numel() * 4

    macs_a, macs_b = case_macs(CASE_A), case_macs(CASE_B)
    bytes_a, bytes_b = case_bytes(CASE_A), case_bytes(CASE_B)
    step_s = total_ms / K / 1e3
    value = job_throughput(2.0 * (macs_a + macs_b), world, step_s)
    peaks, peak_src = load_peaks()
    hbm = peaks["hbm_gbs"]
    fma_peak = fma_peak_tflops(props)
    tf32_peak = peaks["bf16_tflops"] * TF32_OVER_BF16
    tc_rule = tf32_peak / 3.0
    tc_probe = tf32_probe / 3.0 if tf32_probe else None
    ta_s, tb_s = ta_ms / K / 1e3, tb_ms / K / 1e3

    # The algorithms AUTO runs here (the library reports its own choice).
    algo_a = fcv.conv2d_auto_algo(CASE_A.N, CASE_A.Cin, CASE_A.H, CASE_A.W, CASE_A.Cout, CASE_A.P)
    algo_b = fcv.dwsep_conv1d_auto_algo(xb_d, dwb_d, pwb_d, CASE_B.stride, CASE_B.pad)
    tc_a = algo_a in (fcv.CONV2D_TC_3XTF32, fcv.CONV2D_TC_SHIFT_3XTF32)
    tc_b = algo_b in (fcv.CONV1D_TC_3XTF32, fcv.CONV1D_TC_TMA_3XTF32, fcv.CONV1D_TC2_3XTF32)

    def op_entry(c, algo, tensor, t_s, samples):
        e = {"workload": c.name, "algo": ALGO_NAMES.get(algo, algo), "ms": t_s * 1e3,
             "ms_stats": stats_ms(samples) if samples else None,
             "gflops": 2 * case_macs(c) / t_s / 1e9, "macs": case_macs(c), "compulsory_bytes": case_bytes(c),
             "roofline_frac_fp32_fma": op_roofline(c, False, None, fma_peak, hbm) / t_s,
             "roofline_frac_3xtf32": op_roofline(c, True, tc_rule, fma_peak, hbm) / t_s,
             "roofline_frac_3xtf32_probe": (op_roofline(c, True, tc_probe, fma_peak, hbm) / t_s
                                            if tc_probe else None),
             "pipe": "3xtf32" if tensor else "fp32_fma"}
        e["roofline_frac"] = e["roofline_frac_3xtf32"] if tensor else e["roofline_frac_fp32_fma"]
        return e

    per_op = {"conv2d": op_entry(CASE_A, algo_a, tc_a, ta_s, la),
              "dwsep_conv1d": op_entry(CASE_B, algo_b, tc_b, tb_s, lb)}
    if rank == 0 and world == 1:
        flush_buf = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=device)  # 256 MB > L2
        for key, c in (("conv2d_small", wl.CONV2D_SMALL), ("dwsep_conv1d_small", wl.CONV1D_SMALL)):
            algo, legs = time_small_case(lib, fcv, c, stream, flush_buf)
            tensor = algo in (fcv.CONV2D_TC_3XTF32, fcv.CONV2D_TC_SHIFT_3XTF32, fcv.CONV1D_TC_3XTF32,
                              fcv.CONV1D_TC_TMA_3XTF32, fcv.CONV1D_TC2_3XTF32)
            e = op_entry(c, algo, tensor, legs["warm_l2"]["median"] / 1e3, None)
            e["ms_stats"] = legs
            e["note"] = "launch-latency bound; reported, no target"
            per_op[key] = e
        del flush_buf
    fma_src = "148 SMs x 128 FP32 FMA lanes x 2 FLOP x 1965 MHz (spec clocks)"
    gemm_src = ("measured bf16 GEMM (MEASURED_PEAKS.json, %.1f TFLOP/s)" if peak_src == "measured" else
                "bf16 GEMM figure of the profiling recipe's fallback (%.1f TFLOP/s; MEASURED_PEAKS.json absent)")
    tc_src = (gemm_src % peaks["bf16_tflops"] + " x nominal TF32/BF16 (1.1/2.25), / 3 for the three TF32 "
              "products of the 3xTF32 split; FLOPs are the fp32 method's (2 per MAC)")
    tc_probe_src = ("tcgen05.mma kind::tf32 M128 N256 K8 rate probed on this GPU at the start of this run "
                    "(libfcv_probes.so), / 3")
    dom = "conv2d" if ta_s >= tb_s else "dwsep_conv1d"
    if dom == "conv2d":
        achieved = 2 * macs_a / ta_s / 1e12
        if tc_a:
            if algo_a == fcv.CONV2D_TC_SHIFT_3XTF32:
                kname, tkey = "c2s::conv2d_tcs_kernel<4, 1, sum>", "conv2d_tcs_p4"
            else:
                kname = ("c2tc::conv2d_tc4_kernel<4, sum>" if CASE_A.Cout <= 96 and CASE_A.W % 4 == 0
                         else "c2tc::conv2d_tc_kernel<4, sum>")
                tkey = "conv2d_tc_p4"
            roof = {"kernel": kname, "bound": "tensor", "achieved": achieved, "peak": tc_rule, "unit": "TFLOP/s",
                    "frac": achieved / tc_rule, "traffic": traffic_per_launch(tkey), "peak_source": tc_src,
                    "peak_probe": tc_probe, "frac_probe": achieved / tc_probe if tc_probe else None,
                    "peak_probe_source": tc_probe_src}
        else:
            roof = {"kernel": "conv2d_direct_kernel<4, sum>", "bound": "alu", "achieved": achieved,
                    "peak": fma_peak, "unit": "TFLOP/s", "frac": achieved / fma_peak,
                    "traffic": traffic_per_launch("conv2d_direct_p4"), "peak_source": fma_src}
    else:
        if tc_b:
            pw_macs_b = macs_conv1d_pointwise(CASE_B.N, CASE_B.C, CASE_B.T, CASE_B.O, CASE_B.K, CASE_B.stride,
                                              CASE_B.pad)
            achieved = 2 * pw_macs_b / tb_s / 1e12
            if algo_b == fcv.CONV1D_TC2_3XTF32:
                kname, tkey = "tc2::dwsep_conv1d_tc2_kernel<9, 0, 1>", "dwsep_conv1d_tc2"
            else:
                kname, tkey = "tcx::dwsep_conv1d_tcx_kernel<9, 0, 1, 256>", "dwsep_conv1d"
            roof = {"kernel": kname, "bound": "tensor", "achieved": achieved,
                    "peak": tc_rule, "unit": "TFLOP/s", "frac": achieved / tc_rule,
                    "traffic": traffic_per_launch(tkey), "peak_source": tc_src,
                    "achieved_basis": "pointwise MACs (the depthwise MACs run on the FMA pipe)",
                    "peak_probe": tc_probe, "frac_probe": achieved / tc_probe if tc_probe else None}
        else:
            achieved = 2 * macs_b / tb_s / 1e12
            roof = {"kernel": "dwsep_conv1d_fma_kernel", "bound": "alu", "achieved": achieved, "peak": fma_peak,
                    "unit": "TFLOP/s", "frac": achieved / fma_peak, "traffic": None, "peak_source": fma_src}

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": workload_name(), "l2": "inputs larger than L2 (x 604 MB and 134 MB, out 268 MB); "
                   "no flush", "parallelism": f"replicas x{world} (independent batches, no collective)",
                   "algos": {"conv2d": ALGO_NAMES.get(algo_a, algo_a),
                             "dwsep_conv1d": ALGO_NAMES.get(algo_b, algo_b)}},
        "per_op": per_op, "roofline": roof,
        "peaks": {"hbm_gbs": hbm, "fp32_fma_tflops": fma_peak, "tf32_tflops": tf32_peak,
                  "tf32_tflops_probe": tf32_probe, "source": peak_src},
        "e2e": {"value": job_throughput(2.0 * (macs_a + macs_b), world, e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "steps": e2e_steps,
                "overlap": "one stream per op, two step parities (four streams); copies not waited for per call; "
                           "the timed steps include one pipeline fill and drain"},
        # op A: one launch per block of 64 output channels on the shifted-operand kernel, else one; op B: one
        "gpu_launches": K * (((CASE_A.Cout + 63) // 64 if algo_a == fcv.CONV2D_TC_SHIFT_3XTF32 else 1) + 1),
        "clocks": clocks,
        "host": {"cpu_model": cpu_model(), "cores": len(os.sched_getaffinity(0))},
        "source": source_info(),
    }
    if rank == 0 and world == 1:
        # The library's other algorithms on the same inputs (not part of the step).
        def alt_a():
            st = lib.fcv_conv2d_pool_sigmoid_sum_ex(P(xa_d.data_ptr()), P(wa_d.data_ptr()), P(ba_d.data_ptr()),
                                                    CASE_A.N, CASE_A.Cin, CASE_A.H, CASE_A.W, CASE_A.Cout, CASE_A.P,
                                                    P(out_a.data_ptr()), fcv.CONV2D_POOLFIRST, P(sp))
            if st:
                raise fcv.FcvError(st, "pool-first conv2d")

        def alt_b(algo):
            def fn():
                st = lib.fcv_dwsep_conv1d_ex(P(xb_d.data_ptr()), P(dwb_d.data_ptr()), P(pwb_d.data_ptr()),
                                             P(bb_d.data_ptr()), CASE_B.N, CASE_B.C, CASE_B.T, CASE_B.O, CASE_B.K,
                                             CASE_B.stride, CASE_B.pad, P(out_b.data_ptr()), algo, P(sp))
                if st:
                    raise fcv.FcvError(st, f"conv1d algorithm {algo}")
            return fn

        def alt_a_algo(algo):
            def fn():
                st = lib.fcv_conv2d_pool_sigmoid_sum_ex(P(xa_d.data_ptr()), P(wa_d.data_ptr()), P(ba_d.data_ptr()),
                                                        CASE_A.N, CASE_A.Cin, CASE_A.H, CASE_A.W, CASE_A.Cout,
                                                        CASE_A.P, P(out_a.data_ptr()), algo, P(sp))
                if st:
                    raise fcv.FcvError(st, f"conv2d algorithm {algo}")
            return fn

        ta2 = _event_ms(alt_a, 10, stream)
        ta3 = _event_ms(alt_a_algo(fcv.CONV2D_DIRECT), 10, stream)
        ta4 = _event_ms(alt_a_algo(fcv.CONV2D_TC_3XTF32), 10, stream)
        tb = {name: _event_ms(alt_b(algo), 10, stream)
              for name, algo in (("dwsep_conv1d_fma", fcv.CONV1D_FMA),
                                 ("dwsep_conv1d_tc_register_halo", fcv.CONV1D_TC_3XTF32),
                                 ("dwsep_conv1d_tc_tma_halo", fcv.CONV1D_TC_TMA_3XTF32),
                                 ("dwsep_conv1d_2sm", fcv.CONV1D_TC2_3XTF32))}
        pf_macs = CASE_A.N * ((CASE_A.H - 2) // CASE_A.P) * ((CASE_A.W - 2) // CASE_A.P) * CASE_A.Cout * CASE_A.Cin * 9
        result["variants"] = {
            "conv2d_poolfirst": {"ms": ta2, "executed_macs": pf_macs,
                                 "executed_gflops": 2.0 * pf_macs / (ta2 / 1e3) / 1e9,
                                 "speedup_vs_direct": ta_s * 1e3 / ta2,
                                 "note": "pools the input first (exact identity): 9*Cin MACs per pooled value"},
            "conv2d_direct_fma": {"ms": ta3, "gflops": 2.0 * macs_a / (ta3 / 1e3) / 1e9,
                                  "frac_of_fp32_fma_peak": 2.0 * macs_a / (ta3 / 1e3) / 1e12 / fma_peak},
            "conv2d_tc_im2col_3xtf32": {"ms": ta4, "gflops": 2.0 * macs_a / (ta4 / 1e3) / 1e9,
                                        "note": "im2col rows in tensor memory, M = 128 positions, N = Cout"},
        }
        for name, ms in tb.items():
            result["variants"][name] = {"ms": ms, "gflops": 2.0 * macs_b / (ms / 1e3) / 1e9}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["unfused_gpu_baselines"] = unfused_baselines(xa_d, wa_d, ba_d, xb_d, dwb_d, pwb_d, bb_d)
        result["cpu_baseline"] = run_oracle_sample()
    if use_dist:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ----------------------------------------------------------------------------
# unfused GPU baselines (context only; never part of the library)
# ----------------------------------------------------------------------------

def _event_ms(fn, iters, stream):
    """Average device time of fn() over `iters` calls, CUDA events on `stream`."""
    for _ in range(3):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(iters):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def unfused_baselines(xa, wa, ba, xb, dwb, pwb, bb, iters=5):
    """PyTorch eager (cuDNN/cuBLAS) versions of both ops with the intermediates in
    HBM, fp32 with TF32 disabled -- the unfused pipelines the fused kernels replace."""
    import torch.nn.functional as F
    stream = torch.cuda.current_stream()
    prev = (torch.backends.cudnn.allow_tf32, torch.backends.cuda.matmul.allow_tf32)
    torch.backends.cudnn.allow_tf32 = False
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        def op_a():
            y = F.conv2d(xa, wa, ba)
            return torch.sigmoid(F.avg_pool2d(y, CASE_A.P)).sum(dim=(1, 2, 3))

        def op_b():
            d = F.conv1d(xb, dwb.view(CASE_B.C, 1, CASE_B.K), stride=CASE_B.stride, padding=CASE_B.pad,
                         groups=CASE_B.C)
            return F.conv1d(d, pwb.view(CASE_B.O, CASE_B.C, 1), bb)

        ta = _event_ms(op_a, iters, stream)
        tb = _event_ms(op_b, iters, stream)
    finally:
        torch.backends.cudnn.allow_tf32, torch.backends.cuda.matmul.allow_tf32 = prev
    return {"torch_eager_conv2d_pool_sigmoid_sum_ms": ta, "torch_eager_dwsep_conv1d_ms": tb,
            "precision": "fp32, TF32 disabled", "note": "unfused: conv output / depthwise output in HBM"}


def run_probes():
    """Peak probes of libfcv_probes.so on this GPU: FP32 FMA (scalar and packed)
    and the tcgen05 TF32 MMA rate by N, A source and accumulator chains."""
    import ctypes
    from direct_convolution_chip_b200 import build as fcv_build
    torch.cuda.set_device(0)
    lib = ctypes.CDLL(fcv_build.build_probes())
    D = ctypes.c_double
    for packed in (0, 1):
        f, ms = D(), D()
        st = lib.fcvprobe_fma_rate(packed, 2, 20000, ctypes.byref(f), ctypes.byref(ms))
        print(json.dumps({"probe": "fp32_fma", "packed": packed, "status": st, "tflops": f.value / 1e12,
                          "ms": ms.value}), flush=True)
    for n in (32, 64, 128, 256):
        for a_tmem in (0, 1):
            for chains in (1, 2, 4):
                for issuers in (1, 2):
                    if issuers * chains * n > 448:
                        continue
                    f, ms, cyc = D(), D(), D()
                    st = lib.fcvprobe_tf32_mma_rate(n, a_tmem, chains, issuers, 24000, ctypes.byref(f),
                                                    ctypes.byref(ms), ctypes.byref(cyc))
                    print(json.dumps({"probe": "tcgen05_tf32_mma", "n": n, "a_tmem": a_tmem, "chains": chains,
                                      "issuers": issuers, "status": st, "tflops": f.value / 1e12, "ms": ms.value,
                                      "cycles_per_mma": cyc.value}), flush=True)
    run_layout_probes(lib)


def run_layout_probes(lib):
    """The tcgen05 kind::tf32 operand facts the shifted-operand conv2d relies
    on: the B address map for K-major and MN-major descriptors without swizzle,
    the TMEM lanes of an M = 64 accumulator, and SM cycles per MMA."""
    import ctypes
    import numpy as np
    buf = (ctypes.c_float * 2048)()
    for b_major, lbo, sbo in ((0, 128, 128), (0, 256, 128), (1, 128, 128), (1, 256, 128)):
        st = lib.fcvprobe_umma_b_map(b_major, lbo, sbo, buf)
        d = np.frombuffer(buf, dtype=np.float32).reshape(8, 256)
        n = np.arange(256)
        kmajor = np.array([4 * n + (k % 4) + (lbo // 4) * (k // 4) for k in range(8)])  # rows 16 B apart
        mnmajor = np.array([(n % 4) + (sbo // 4) * (n // 4) + 4 * k for k in range(8)])
        print(json.dumps({"probe": "umma_b_map", "b_major": b_major, "lbo": lbo, "sbo": sbo, "status": st,
                          "all_zero": bool(np.all(d == 0)),
                          "matches_k_major_rows_16B": bool(np.array_equal(d, kmajor % 2048)),
                          "matches_mn_major_interleave": bool(np.array_equal(d, mnmajor % 2048)),
                          "k0_n0_7": d[0, :8].astype(int).tolist(), "k4_n0_7": d[4, :8].astype(int).tolist()}),
              flush=True)
    rows = (ctypes.c_float * 128)()
    st = lib.fcvprobe_umma_m64_rows(rows)
    r = np.frombuffer(rows, dtype=np.float32).astype(int)
    print(json.dumps({"probe": "umma_m64_rows", "status": st,
                      "lanes_written": [int(i) for i in np.nonzero(r != -7)[0]],
                      "row_of_lane": {int(i): int(r[i]) - 1 for i in np.nonzero(r != -7)[0]}}), flush=True)
    for m, n, a_tmem in ((128, 256, 0), (128, 256, 1), (64, 256, 1), (128, 192, 1), (64, 192, 1)):
        best = None
        for _ in range(3):
            c = ctypes.c_double()
            st = lib.fcvprobe_umma_cycles(m, n, a_tmem, 2000, ctypes.byref(c))
            best = c.value if best is None else min(best, c.value)
        print(json.dumps({"probe": "umma_cycles", "m": m, "n": n, "a": "tmem" if a_tmem else "smem",
                          "b": "smem, K-major, no swizzle", "status": st, "sm_cycles_per_mma": best}), flush=True)
    # Swizzled K-major B with shifted start addresses (the column taps of the
    # shifted-operand conv2d): which word each (k, n) reads, under two readings
    # of the swizzle -- on the matrix-relative row, or on the absolute address.
    n = np.arange(256)
    for layout, row_bytes, starts in ((6, 32, (0, 128, 256, 384)), (4, 64, (0, 256, 512))):
        atom = 8 * row_bytes
        for start in starts:
            for base_off in sorted({0, (start >> 7) & 7}):
                st = lib.fcvprobe_umma_b_map_ex(layout, 16, atom, start, base_off, buf)
                d = np.frombuffer(buf, dtype=np.float32).reshape(8, 256).astype(np.int64)
                rel, ab = [], []
                chunks = row_bytes // 16  # 16-byte chunks per row; the swizzle XORs their index
                for k in range(8):
                    off = start + (n // 8) * atom + (n % 8) * row_bytes
                    swz_rel = (((n % 8) * row_bytes) >> 7) & (chunks - 1)  # from the row inside the matrix
                    swz_abs = (off >> 7) & (chunks - 1)                      # from the shared-memory address
                    rel.append((off + ((k // 4) ^ swz_rel) * 16 + (k % 4) * 4) // 4)
                    ab.append((off + ((k // 4) ^ swz_abs) * 16 + (k % 4) * 4) // 4)
                rel, ab = np.array(rel) % 2048, np.array(ab) % 2048
                print(json.dumps({"probe": "umma_b_map_swizzled", "layout": {6: "SW32", 4: "SW64"}[layout],
                                  "start_offset": start, "base_offset": base_off, "status": st,
                                  "matches_relative_row_swizzle": bool(np.array_equal(d, rel)),
                                  "matches_absolute_address_swizzle": bool(np.array_equal(d, ab)),
                                  "k0_n0_7": d[0, :8].tolist(), "k4_n0_7": d[4, :8].tolist()}), flush=True)
    for name, layout, lbo, sbo, shift in (("none, planes 3200 B apart, rows 16 B (conv2d today)", 0, 3200, 128, 64),
                                          ("SW32, rows 32 B", 6, 16, 256, 128), ("SW32, rows 32 B, no shift", 6, 16, 256, 0),
                                          ("SW64, rows 64 B", 4, 16, 512, 256)):
        best = None
        for _ in range(3):
            c = ctypes.c_double()
            st = lib.fcvprobe_umma_cycles_ex(128, 192, 1, layout, lbo, sbo, shift, 2001, ctypes.byref(c))
            best = c.value if best is None else min(best, c.value)
        print(json.dumps({"probe": "umma_cycles_shifted_b", "m": 128, "n": 192, "a": "tmem", "b": name,
                          "start_shift_bytes": shift, "status": st, "sm_cycles_per_mma": best}), flush=True)


def run_configs(args):
    """One JSON line per workload (named configs and the 48-point sweep): the
    metric per config, GFLOP/s and fraction of its roofline."""
    import ctypes
    import direct_convolution_chip_b200 as fcv
    torch.cuda.set_device(0)
    lib = fcv.load()
    P = ctypes.c_void_p
    props = torch.cuda.get_device_properties(0)
    peaks, _ = load_peaks()
    fma_peak = fma_peak_tflops(props)
    tf32_peak = peaks["bf16_tflops"] * TF32_OVER_BF16
    tf32_probe = probe_tf32_tflops()  # the on-box tcgen05 TF32 rate, for the second fraction
    stream = torch.cuda.current_stream()
    sp = P(stream.cuda_stream)
    cases = list(wl.NAMED) + (wl.sweep_cases() if args.sweep else [])
    for c in cases:
        if c.op == "conv2d":
            x, w, b = [t.cuda() for t in wl.conv2d_inputs(c)]
            out = torch.empty((c.N,), device="cuda")
            fn = lambda: lib.fcv_conv2d_pool_sigmoid_sum(P(x.data_ptr()), P(w.data_ptr()), P(b.data_ptr()), c.N,
                                                         c.Cin, c.H, c.W, c.Cout, c.P, P(out.data_ptr()), sp)
            algo = fcv.conv2d_auto_algo(c.N, c.Cin, c.H, c.W, c.Cout, c.P)
            tc = algo in (fcv.CONV2D_TC_3XTF32, fcv.CONV2D_TC_SHIFT_3XTF32)
            pipe, peak = ("3xtf32", tf32_peak / 3.0) if tc else ("fp32_fma", fma_peak)
        else:
            x, dw, pw, b = [t.cuda() for t in wl.conv1d_inputs(c)]
            To = (c.T + 2 * c.pad - c.K) // c.stride + 1
            out = torch.empty((c.N, c.O, To), device="cuda")
            fn = lambda: lib.fcv_dwsep_conv1d(P(x.data_ptr()), P(dw.data_ptr()), P(pw.data_ptr()), P(b.data_ptr()),
                                              c.N, c.C, c.T, c.O, c.K, c.stride, c.pad, P(out.data_ptr()), sp)
            algo = fcv.dwsep_conv1d_auto_algo(x, dw, pw, c.stride, c.pad)
            tc = algo != fcv.CONV1D_FMA
            pipe, peak = ("3xtf32", tf32_peak / 3.0) if tc else ("fp32_fma", fma_peak)
        assert fn() == 0
        macs, nbytes = case_macs(c), case_bytes(c)
        iters = max(3, min(200, int(0.2 / max(2.0 * macs / (peak * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)))))
        ms = _event_ms(fn, iters, stream)
        roof_macs = macs if (pipe == "fp32_fma" or c.op == "conv2d") else \
            macs_conv1d_pointwise(c.N, c.C, c.T, c.O, c.K, c.stride, c.pad)
        roof = roofline_time_s(roof_macs, nbytes, peak, peaks["hbm_gbs"])
        line = {"config": c.name, "op": c.op, "algo": ALGO_NAMES.get(algo, algo), "ms": ms,
                "gflops": 2.0 * macs / (ms / 1e3) / 1e9,
                "macs": macs, "bytes": nbytes, "pipe": pipe, "roofline_ms": roof * 1e3,
                "roofline_frac": roof / (ms / 1e3), "l2": "inputs resident; no flush"}
        if pipe == "3xtf32" and tf32_probe:
            roof_p = roofline_time_s(roof_macs, nbytes, tf32_probe / 3.0, peaks["hbm_gbs"])
            line["roofline_frac_3xtf32_probe"] = roof_p / (ms / 1e3)
        print(json.dumps(line), flush=True)
        del x, out


# ----------------------------------------------------------------------------
# the reference arm: the CPU oracle on a bounded sample per step
# ----------------------------------------------------------------------------

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    xa, wa, ba = wl.conv2d_inputs(CASE_A)
    xb, dwb, pwb, bb = wl.conv1d_inputs(CASE_B)
    xa, wa, ba = xa.numpy(), wa.numpy(), ba.numpy()
    xb, dwb, pwb, bb = xb.numpy(), dwb.numpy(), pwb.numpy(), bb.numpy()
    # Per step: one batch item of each op, restricted to the first m output
    # channels so that warm-up + timed steps end within a few minutes.
    budget = min(1.5, 150.0 / max(1, args.steps + args.warmup))

    def step(i, ca, cb):
        na, nb = i % CASE_A.N, i % CASE_B.N
        oracle.conv2d_pool_sigmoid_sum(xa[na:na + 1], wa[:ca], ba[:ca], CASE_A.P)
        oracle.dwsep_conv1d(xb[nb:nb + 1], dwb, pwb[:cb], bb[:cb], CASE_B.stride, CASE_B.pad)

    t = time.perf_counter()
    step(0, 4, 16)
    t1 = time.perf_counter() - t
    scale = max(1.0, budget / max(t1, 1e-4))
    ca = int(min(CASE_A.Cout, max(1, 4 * scale)))
    cb = int(min(CASE_B.O, max(1, 16 * scale)))
    for i in range(args.warmup):
        step(i, ca, cb)
    t = time.perf_counter()
    for i in range(args.steps):
        step(i, ca, cb)
    dt = time.perf_counter() - t
    macs = (macs_conv2d(1, CASE_A.Cin, CASE_A.H, CASE_A.W, ca, CASE_A.P)
            + macs_conv1d(1, CASE_B.C, CASE_B.T, cb, CASE_B.K, CASE_B.stride, CASE_B.pad))
    value = 2.0 * macs * args.steps / dt / 1e9
    full_macs = (macs_conv2d(CASE_A.N, CASE_A.Cin, CASE_A.H, CASE_A.W, CASE_A.Cout, CASE_A.P)
                 + macs_conv1d(CASE_B.N, CASE_B.C, CASE_B.T, CASE_B.O, CASE_B.K, CASE_B.stride, CASE_B.pad))
    sample = (f"per step: op A on 1 batch item with {ca} of {CASE_A.Cout} output channels, op B on 1 batch "
              f"item with {cb} of {CASE_B.O} output channels")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(), "parallelism": "CPU oracle, rank 0 only", "sample": sample,
                   "sampled_fraction_of_step": macs / full_macs},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_profile(args):
    """Only one fused op, `--steps` times after `--warmup` calls, nothing else
    launched: the target of the committed ncu captures.  `--batch` replaces the
    batch size (a smaller case for full-section captures), `--algo` the
    algorithm (default AUTO)."""
    import direct_convolution_chip_b200 as fcv
    import dataclasses
    torch.cuda.set_device(0)
    c = CASE_A if args.profile == "conv2d" else CASE_B
    if args.batch:
        c = dataclasses.replace(c, N=args.batch, name=f"{c.name}_n{args.batch}")
    algo = args.algo
    if c.op == "conv2d":
        x, w, b = [t.cuda() for t in wl.conv2d_inputs(c)]
        out = torch.empty((c.N,), device="cuda")
        fn = lambda: fcv.conv2d_pool_sigmoid_sum(x, w, b, c.P, out=out, algo=algo)
    else:
        x, dw, pw, b = [t.cuda() for t in wl.conv1d_inputs(c)]
        To = (c.T + 2 * c.pad - c.K) // c.stride + 1
        out = torch.empty((c.N, c.O, To), device="cuda")
        fn = lambda: fcv.dwsep_conv1d(x, dw, pw, b, c.stride, c.pad, out=out, algo=algo)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"profile": c.name, "algo": algo, "steps": args.steps,
                      "ms_per_call": e0.elapsed_time(e1) / args.steps, "device_error": fcv.device_error()}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["fcv", "reference"], default="fcv")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle and unfused-baseline legs")
    ap.add_argument("--configs", action="store_true", help="time every named workload, one JSON line each")
    ap.add_argument("--sweep", action="store_true", help="with --configs: the 48-point shape sweep as well")
    ap.add_argument("--probe", action="store_true",
                    help="run the FP32-FMA and tcgen05 TF32 peak probes, one JSON line each")
    ap.add_argument("--profile", choices=["conv2d", "dwsep_conv1d"],
                    help="run only this op of the step (the target of ncu captures)")
    ap.add_argument("--batch", type=int, default=0, help="with --profile: batch size instead of the full one")
    ap.add_argument("--algo", type=int, default=0, help="with --profile: algorithm selector (0: AUTO)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    elif args.probe:
        run_probes()
    elif args.profile:
        run_profile(args)
    elif args.configs:
        run_configs(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
