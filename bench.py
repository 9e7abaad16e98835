"""WBMM benchmark on B200: TFLOP/s, HBM GB/s and fraction of roofline.

One step is one pass of the operator's hot path over one batch of seeded
synthetic input.  Default workload (the training step): B128 C256 28x28, w=14,
bf16 -- forward y = WBMM(x; T), then the backward dX = M^T dY and the table
gradient dT, all through the C ABI.  Other workloads (--workload): fwd
(B64 C128 56x56 w14), sweep7 / sweep14 / sweep28 (B32 C256 112x112), cached
(B8 C96 224x224 w14, cached matrices + 3x3 mixing), fwd32 / train32 / cached32
(the fp32 path on the fwd, train and cached shapes) and reparam (the cached
shape through one matrix merged from a 14x14 and a 7x7 table).

Multi-GPU (torchrun): every rank owns its own block of channels with the
per-GPU workload above (weak scaling); channels are independent, so the hot
path has no collective.  Timing is device time (CUDA events) with a barrier on
both sides, max over ranks.

--impl reference runs the fp64 CPU oracle on the host cores instead (bounded
sample per step), a deliberately slow comparison arm with the same JSON line.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "WBMM fwd/bwd TFLOP/s, HBM GB/s and % of roofline at w=14 bf16 on 1 B200"
L2_BYTES = 126 * 2 ** 20

WORKLOADS = {
    "train": "train_bf16",
    "fwd": "fwd_bf16",
    "fwd32": "fwd_f32",
    "train32": "train_f32",
    "cached32": "hires_cached_dw_f32",
    "sweep7": "sweep_w7",
    "sweep14": "sweep_w14",
    "sweep28": "sweep_w28",
    "cached": "hires_cached_dw",
    "reparam": "hires_reparam",
}


def fp32_fma_peak_tflops(dev):
    """CUDA-core fp32 peak: 128 fp32 lanes per SM, one FMA (2 FLOP) per lane
    per cycle, at the B200's 1965 MHz maximum SM clock."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return sms * 128 * 2 * 1.965e9 / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------ workload math

def step_flops(wl):
    n = wl.B * wl.C * wl.H * wl.W
    f = 2.0 * n * wl.d
    if wl.kind == "train":
        return 3 * f
    if wl.kind == "cached_dw":
        return f + 18.0 * n
    return f


def step_bytes(wl):
    """Algorithmic bytes: each tensor of the step read or written once."""
    e = 2 if wl.dtype == "bf16" else 4
    m = wl.B * wl.C * wl.H * wl.W * e
    tbl = wl.C * wl.t * e
    if wl.kind == "train":
        return 5 * m + tbl + wl.C * wl.t * 4          # x, y, dY, x, dX, T, dT
    if wl.kind == "cached_dw":
        return 2 * m + wl.C * wl.d * wl.d * e + wl.C * 9 * e   # x, z, M, K
    if wl.kind == "reparam":
        return 2 * m + wl.C * wl.d * wl.d * e                  # x, y, merged M
    return 2 * m + tbl


def kernel_bytes(wl, name):
    e = 2 if wl.dtype == "bf16" else 4
    m = wl.B * wl.C * wl.H * wl.W * e
    tbl = wl.C * wl.t * e
    return {"forward": 2 * m + tbl, "backward_dx": 2 * m + tbl,
            "backward_dt": 2 * m + wl.C * wl.t * 4,
            # x, dY (once), dX, T, dT: both gradients in one call
            "backward": 3 * m + tbl + wl.C * wl.t * 4,
            "forward_cached": 2 * m + wl.C * wl.d * wl.d * e,
            "forward_cached_dw3x3": 2 * m + wl.C * wl.d * wl.d * e + wl.C * 9 * e,
            # the merged matrix written, both tables read
            "reparam_merge": wl.C * wl.d * wl.d * e + tbl
                             + wl.C * (2 * synth.REPARAM_SMALL_WINDOW - 1) ** 2 * e,
            "dw3x3": 2 * m + wl.C * 9 * e}[name]


def kernel_flops(wl, name):
    n = wl.B * wl.C * wl.H * wl.W
    if name == "dw3x3":
        return 18.0 * n
    if name == "forward_cached_dw3x3":
        return 2.0 * n * wl.d + 18.0 * n
    if name == "reparam_merge":
        return float(wl.C * wl.d * wl.d)
    if name == "backward":
        return 4.0 * n * wl.d
    return 2.0 * n * wl.d


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="wbmm_clocks_gpu%d_" % self.gpu, suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- GPU arm

class Arm:
    """Device buffers and the step of one workload (one rank)."""

    def __init__(self, wl, seed, nsets, dev, fused=False):
        import windowed_matmul_conv_b200 as wb
        self.wb = wb
        self.wl = wl
        # cached bf16 workloads: the step is the fused cached forward + 3x3
        self.fused = fused and wl.kind == "cached_dw" and wl.dtype == "bf16"
        self.dev = dev
        d = synth.draw(wl, seed=seed)
        self.host = d
        self.sets = []
        for k in range(nsets):
            s = {"x": d["x"].to(dev)}
            if k > 0:   # distinct bytes per set so that no set is an L2 copy of another
                s["x"] = torch.roll(s["x"], shifts=k, dims=0).contiguous()
            s["y"] = torch.empty_like(s["x"])
            if wl.kind == "train":
                s["dY"] = torch.roll(d["dY"].to(dev), shifts=k, dims=0).contiguous()
                s["dX"] = torch.empty_like(s["x"])
            self.sets.append(s)
        self.T = d["T"].to(dev)
        if wl.kind == "train":
            self.dT = torch.empty((wl.C, wl.t), dtype=torch.float32, device=dev)
            nbytes = wb.wbmm_backward_workspace_bytes(wl.B, wl.C, wl.H, wl.W, wl.w,
                                                      synth.torch_dtype(wl.dtype))
            # zero-filled once: the table gradient's arrival counters start at zero
            self.ws = torch.zeros(max(1, nbytes // 4), dtype=torch.float32, device=dev)
        if wl.kind == "reparam":
            self.Tk = d["Tk"].to(dev)
            self.M = wb.reparam_merge(self.T, self.Tk, wl.w, synth.REPARAM_SMALL_WINDOW)
            self.M2 = torch.empty_like(self.M)     # target of the timed merges
        if wl.kind == "cached_dw":
            self.M = wb.cache_matrices(self.T, wl.w)
            self.K = d["K"].to(dev)
            for s in self.sets:
                s["z"] = torch.empty_like(s["x"])

    def kernels(self):
        """The step's launch units, one call each (the per-call breakdown).
        The training step's backward call launches the input-gradient and
        table-gradient kernels side by side on disjoint SMs; it is timed as
        one unit."""
        k = self.wl.kind
        if k == "train":
            return ["forward", "backward"]
        if k == "cached_dw":
            return ["forward_cached_dw3x3"] if self.fused else ["forward_cached", "dw3x3"]
        if k == "reparam":
            return ["forward_cached"]
        return ["forward"]

    def alternatives(self):
        """Other launches of the same step, timed for reference only: the
        fused cached forward + 3x3 (one launch; slower than the two calls on
        224x224 planes, where its CUDA-core stencil costs more per tile than
        the HBM time it saves), or the two calls when --fused makes the
        fused launch the step."""
        if self.wl.kind == "reparam":
            return ["reparam_merge"]    # one-time preparation of the inference matrix
        if self.wl.kind == "train":
            # one gradient per call: each kernel alone on the whole device
            return ["backward_dx", "backward_dt"]
        # the fused launch covers bf16 maps only
        if self.wl.kind == "cached_dw" and self.wl.dtype == "bf16":
            return ["forward_cached", "dw3x3"] if self.fused else ["forward_cached_dw3x3"]
        return []

    def calls(self):
        """The step as a user issues it: the training step is one forward
        and one backward call that returns both dX and dT."""
        return self.kernels()

    def launch(self, name, s):
        wb, w = self.wb, self.wl.w
        if name == "forward":
            wb.wbmm_forward(s["x"], self.T, s["y"], w)
        elif name == "backward_dx":
            wb.wbmm_backward(None, self.T, s["dY"], s["dX"], None, None, w)
        elif name == "backward_dt":
            wb.wbmm_backward(s["x"], None, s["dY"], None, self.dT, self.ws, w)
        elif name == "backward":
            wb.wbmm_backward(s["x"], self.T, s["dY"], s["dX"], self.dT, self.ws, w)
        elif name == "forward_cached":
            wb.wbmm_forward_cached(s["x"], self.M, None, s["y"], w)
        elif name == "forward_cached_dw3x3":
            wb.wbmm_forward_cached(s["x"], self.M, self.K, s["z"], w)
        elif name == "reparam_merge":
            wb.wbmm_reparam_merge(self.T, self.Tk, self.M2, w, synth.REPARAM_SMALL_WINDOW)
        elif name == "dw3x3":
            wb.wbmm_dw3x3(s["y"], self.K, s["z"])

    def step(self, k):
        s = self.sets[k % len(self.sets)]
        for name in self.calls():
            self.launch(name, s)


def barrier(world):
    if world > 1:
        dist.barrier()


def max_over_ranks(v, world, dev):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v, world, dev):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def prefill(ms=20.0):
    """Keeps the GPU busy while the host enqueues the timed launches."""
    torch.cuda._sleep(int(ms * 1e6 * 2.0))   # ~2 GHz cycles per ns


def kernel_source_hash(source):
    """sha256 (16 hex digits) of a kernel source file followed by the local
    headers it includes (csrc/*.cuh and *.h, in include order), so that a
    change to shared device code also invalidates a recorded capture."""
    import hashlib
    import re
    path = os.path.join(ROOT, source)
    h = hashlib.sha256()
    with open(path, "rb") as f:
        text = f.read()
    h.update(text)
    for inc in re.findall(rb'#include "([^"]+)"', text):
        hp = os.path.join(os.path.dirname(path), inc.decode())
        if os.path.exists(hp):
            with open(hp, "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from the committed ncu capture, or None when the
    kernel source changed since the counters were taken.  The backward call
    is the sum of its two kernels' captures (ncu runs them one after the
    other, so the second read of dY counts again)."""
    if kernel == "backward":
        parts = [recorded_traffic("backward_dx"), recorded_traffic("backward_dt")]
        return None if None in parts else sum(parts)
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(kernel)
        if not rec:
            return None
        return rec["bytes"] if kernel_source_hash(rec["source"]) == rec["sha256_16"] else None
    except (OSError, ValueError, KeyError):
        return None


def cpu_baseline(wl, host, budget_s=10.0):
    """The oracle, as it stands, on a bounded sample: the first images of the
    same inputs (all channels), repeated until `budget_s` of CPU time."""
    import oracle
    bs = max(1, min(wl.B, 32 if wl.kind == "train" else 8))
    sub = wl.scaled(B=bs)
    x = host["x"][:bs]
    T = host["T"]
    runs, t0 = 0, time.perf_counter()
    while True:
        if wl.kind == "train":
            dy = host["dY"][:bs]
            oracle.forward(x, T, wl.w)
            oracle.backward_dx(dy, T, wl.w)
            oracle.backward_dt(x, dy, wl.w)
        elif wl.kind == "cached_dw":
            M = oracle.expand(T, wl.w)
            y = oracle.forward_cached(x, M, wl.w)
            oracle.dw3x3(y, host["K"])
        elif wl.kind == "reparam":
            M = oracle.reparam_merge(T, host["Tk"], wl.w, synth.REPARAM_SMALL_WINDOW)
            oracle.forward_cached(x, M, wl.w)
        else:
            oracle.forward(x, T, wl.w)
        runs += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    tf = step_flops(sub) * runs / el / 1e12
    return {"value": tf, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d of %d images, all %d channels, %d repetitions, %.1f s (fp64 C loops)"
                      % (bs, wl.B, wl.C, runs, el)}


def workload_label(wl):
    """The workload's name in both arms' JSON lines."""
    what = {"train": "forward + dX + dT", "forward": "forward",
            "cached_dw": "cached forward, then 3x3",
            "reparam": "cached forward with the merged 14x14 + 7x7 matrix"}[wl.kind]
    return "%s: B%d C%d %dx%d w%d (%s)" % (wl.name, wl.B, wl.C, wl.H, wl.W, wl.w, what)


def dw5x5_context(sets, K, stream):
    """Same-run context, not part of the step: torch's depthwise 5x5
    convolution (padding 2, library kernel) on the step's input maps, the
    baseline the pages compare WBMM with.  Never raises: a failure is
    reported in the returned record."""
    rec = {"op": "torch conv2d, 5x5 depthwise (groups=C), padding 2, on the step's x"}
    try:
        xs = [s["x"] for s in sets]
        C = xs[0].shape[1]
        g = torch.Generator(device="cpu")
        g.manual_seed(5)
        wgt = (torch.randn((C, 1, 5, 5), generator=g) * 0.2).to(xs[0].dtype).to(xs[0].device)
        with torch.no_grad():
            for k in range(3):
                torch.nn.functional.conv2d(xs[k % len(xs)], wgt, padding=2, groups=C)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for k in range(K):
                torch.nn.functional.conv2d(xs[k % len(xs)], wgt, padding=2, groups=C)
            b.record(stream)
            torch.cuda.synchronize()
        us = a.elapsed_time(b) / K * 1e3
        nbytes = 2 * xs[0].numel() * xs[0].element_size()
        rec.update({"us": round(us, 2), "gbs": round(nbytes / (us * 1e-6) / 1e9, 1)})
    except Exception as e:   # context only: never costs the benchmark line
        rec["unavailable"] = ("%s: %s" % (type(e).__name__, e))[:200]
    return rec


def e2e_pipelined(arm, host_in, host_out, ke, stream):
    """ms per step of ``ke`` steps through the public API with host buffers,
    the copies overlapped with the steps: step k runs on buffer set k % 2
    while the inputs of step k+1 are copied in on one stream and the outputs
    of step k-1 are copied out on another (host-to-device and device-to-host
    copies use the link in both directions at once).  Returns None if the
    streams cannot be set up; the caller then reports the serial figure."""
    try:
        sets = arm.sets[:2]
        cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
        in_ev = [torch.cuda.Event() for _ in sets]
        done_ev = [torch.cuda.Event() for _ in sets]
        out_ev = [torch.cuda.Event() for _ in sets]
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        g0.record(stream)
        cin.wait_stream(stream)
        cout.wait_stream(stream)
        for k in range(ke):
            j = k % 2
            s = sets[j]
            with torch.cuda.stream(cin):
                cin.wait_event(done_ev[j])        # step k-2 has read this set's inputs
                for nm, t in host_in.items():
                    s[nm].copy_(t, non_blocking=True)
                in_ev[j].record(cin)
            stream.wait_event(in_ev[j])
            stream.wait_event(out_ev[j])          # this set's outputs of step k-2 are out
            if "dT" in host_out:
                stream.wait_event(out_ev[1 - j])  # dT (one buffer) of step k-1 is out
            arm.step(j)
            done_ev[j].record(stream)
            with torch.cuda.stream(cout):
                cout.wait_event(done_ev[j])
                for nm, t in host_out.items():
                    t.copy_(arm.dT if nm == "dT" else s[nm], non_blocking=True)
                out_ev[j].record(cout)
        stream.wait_stream(cout)
        g1.record(stream)
        torch.cuda.synchronize()
        return g0.elapsed_time(g1) / ke
    except Exception:   # never costs the benchmark line
        try:
            torch.cuda.synchronize()
        except Exception:
            pass
        return None


class GraphSteps:
    """CUDA graphs of an arm's steps: one holding a step on each buffer set in
    turn (the kernels of consecutive steps overlap their prologues and tails
    through programmatic dependent launch, as in a training loop) and one
    single step per set for the remainder of K."""

    def __init__(self, arm):
        self.nsets = len(arm.sets)
        self.all = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.all):
            for k in range(self.nsets):
                arm.step(k)
        self.one = []
        for k in range(self.nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                arm.step(k)
            self.one.append(g)
        self.all.replay()
        for g in self.one:
            g.replay()
        torch.cuda.synchronize()

    def replay(self, K):
        full, rest = divmod(K, self.nsets)
        for _ in range(full):
            self.all.replay()
        for k in range(rest):
            self.one[k].replay()

    def release(self):
        del self.all
        self.one = []


def roofline_of(wl, value_tf, peaks):
    """Fraction of the step's roofline, min(tensor peak, AI x HBM), that the
    step's algorithmic throughput reaches (burst tensor peak; fp32 steps
    against the CUDA-core FMA peak)."""
    top = peaks["bf16_tflops"] if wl.dtype == "bf16" else peaks["fp32_fma_tflops"]
    ai = step_flops(wl) / step_bytes(wl)
    roof = min(top, ai * peaks["hbm_gbs"] / 1e3)
    return {"bound": "tensor" if roof >= top else "hbm", "roofline_tflops": round(roof, 1),
            "frac": round(value_tf / roof, 4)}


# The benchmark's other workloads, timed after the headline step on one GPU
WORKLOAD_SWEEP = ("fwd", "sweep7", "sweep14", "sweep28", "cached")


def time_workloads(dev, peaks, K):
    """Graph-timed device time of every other workload (K steps each after 3
    warm-up steps, 3 rotating buffer sets larger than L2), with the fused
    cached forward + 3x3 timed beside its two-call step.  Never raises: a
    failing workload is reported in its record."""
    out = {}
    for key in WORKLOAD_SWEEP:
        wl = synth.WORKLOADS[WORKLOADS[key]]
        rec = {"workload": workload_label(wl)}
        try:
            arm = Arm(wl, seed=0, nsets=3, dev=dev)
            for k in range(3):
                arm.step(k)
            torch.cuda.synchronize()
            gs = GraphSteps(arm)
            stream = torch.cuda.current_stream()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            prefill(5.0)
            e0.record(stream)
            gs.replay(K)
            e1.record(stream)
            torch.cuda.synchronize()
            gs.release()
            ms = e0.elapsed_time(e1) / K
            tf = step_flops(wl) / (ms * 1e-3) / 1e12
            rec.update({"us": round(ms * 1e3, 2), "tflops": round(tf, 1),
                        "gbs": round(step_bytes(wl) / (ms * 1e-3) / 1e9, 1),
                        "windows_channels_per_s": round(wl.windows_per_channel * wl.C
                                                        / (ms * 1e-3), 1),
                        "calls": arm.calls()})
            rec.update(roofline_of(wl, tf, peaks))
            for name in arm.alternatives():
                s = arm.sets[0]
                for _ in range(3):
                    arm.launch(name, s)
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                a0.record(stream)
                for k in range(K):
                    arm.launch(name, arm.sets[k % len(arm.sets)])
                a1.record(stream)
                torch.cuda.synchronize()
                us = a0.elapsed_time(a1) / K * 1e3
                rec.setdefault("alternatives", {})[name] = {
                    "us": round(us, 2), "gbs": round(kernel_bytes(wl, name) / (us * 1e-6) / 1e9, 1),
                    "frac_of_step_roofline": round(step_flops(wl) / (us * 1e-6) / 1e12
                                                   / rec["roofline_tflops"], 4)}
            assert arm.wb.wbmm_get_device_status() == 0, "device status"
            del arm
        except Exception as e:   # reported, never costs the headline line
            rec["error"] = ("%s: %s" % (type(e).__name__, e))[:200]
        torch.cuda.empty_cache()
        out[key] = rec
    return out


def run_gpu(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[WORKLOADS[args.workload]]
    from windowed_matmul_conv_b200.sharding import channel_range
    peaks = load_peaks()
    peaks["fp32_fma_tflops"] = fp32_fma_peak_tflops(dev)
    wb_arm = Arm(wl, seed=rank, nsets=3, dev=dev, fused=args.fused)
    wb = wb_arm.wb
    K, W = args.steps, args.warmup
    stream = torch.cuda.current_stream()

    # warm-up (also configures kernels before graph capture)
    for k in range(W):
        wb_arm.step(k)
    torch.cuda.synchronize()
    assert wb.wbmm_get_device_status() == 0, "device status after warm-up"

    gsteps = GraphSteps(wb_arm)

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)

    # ---- region A: K steps, device time
    launches0 = wb.wbmm_launch_count()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    prefill()
    e0.record(stream)
    gsteps.replay(K)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_step = ms_total / K
    assert wb.wbmm_launch_count() == launches0   # graphs: no host launches

    # ---- region B: the same steps launched eagerly, events around each kernel
    names = wb_arm.kernels()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in names] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    prefill()
    launches1 = wb.wbmm_launch_count()
    for k in range(K):
        s = wb_arm.sets[k % len(wb_arm.sets)]
        for j, name in enumerate(names):
            evs[k][j][0].record(stream)
            wb_arm.launch(name, s)
            evs[k][j][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    # the graph replays launch the same kernels as these eager steps
    gpu_launches = wb.wbmm_launch_count() - launches1
    alt = {}
    for name in wb_arm.alternatives():
        s = wb_arm.sets[0]
        for _ in range(3):
            wb_arm.launch(name, s)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a0.record(stream)
        for k in range(K):
            wb_arm.launch(name, wb_arm.sets[k % len(wb_arm.sets)])
        a1.record(stream)
        torch.cuda.synchronize()
        us = max_over_ranks(a0.elapsed_time(a1) / K, world, dev) * 1e3
        alt[name] = {"us": round(us, 2),
                     "gbs": round(kernel_bytes(wl, name) / (us * 1e-6) / 1e9, 1)}
    kern = {}
    for j, name in enumerate(names):
        iso = sum(evs[k][j][0].elapsed_time(evs[k][j][1]) for k in range(K)) / K
        iso = max_over_ranks(iso, world, dev)
        # steady state: K calls of this entry point back to back (rotating
        # buffer sets), one event pair around all of them, so that each call
        # overlaps its set-up with the previous call's tail as it does inside
        # the step; the isolated figure (an event pair around each call of
        # the eager step) pays every call's ramp in full
        for _ in range(3):
            wb_arm.launch(name, wb_arm.sets[0])
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        prefill(5.0)
        c0.record(stream)
        for k in range(K):
            wb_arm.launch(name, wb_arm.sets[k % len(wb_arm.sets)])
        c1.record(stream)
        torch.cuda.synchronize()
        avg = max_over_ranks(c0.elapsed_time(c1) / K, world, dev)
        gbs = kernel_bytes(wl, name) / (avg * 1e-3) / 1e9
        kern[name] = {"us": round(avg * 1e3, 2), "gbs": round(gbs, 1),
                      "tflops": round(kernel_flops(wl, name) / (avg * 1e-3) / 1e12, 2),
                      "hbm_frac": round(gbs / peaks["hbm_gbs"], 3),
                      "us_isolated": round(iso * 1e3, 2)}
    clk = clocks.stop()
    assert wb.wbmm_get_device_status() == 0, "device status after timing"

    # ---- e2e: pinned host inputs -> device -> step -> host outputs
    host_in = {"x": wb_arm.host["x"].pin_memory()}
    if wl.kind == "train":
        host_in["dY"] = wb_arm.host["dY"].pin_memory()
    s0 = wb_arm.sets[0]
    outs = (["y"] if wl.kind in ("forward", "reparam")
            else (["y", "dX"] if wl.kind == "train" else ["z"]))
    host_out = {o: torch.empty(s0[o].shape, dtype=s0[o].dtype, pin_memory=True) for o in outs}
    if wl.kind == "train":
        host_out["dT"] = torch.empty(wb_arm.dT.shape, dtype=torch.float32, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    ke = max(2, min(K, 10))
    barrier(world)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for k in range(ke):
        for nm, t in host_in.items():
            s0[nm].copy_(t, non_blocking=True)
        wb_arm.step(0)
        for nm, t in host_out.items():
            src = wb_arm.dT if nm == "dT" else s0[nm]
            t.copy_(src, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, dev) / ke
    # the same steps with the copies pipelined: two buffer sets, the next
    # step's inputs copied in and the previous step's outputs copied out on
    # their own streams while a step computes
    barrier(world)
    pip_ms = e2e_pipelined(wb_arm, host_in, host_out, ke, stream)
    failed = max_over_ranks(1.0 if pip_ms is None else 0.0, world, dev)   # on any rank
    pip_ms = None if failed else max_over_ranks(pip_ms, world, dev)
    barrier(world)

    context = dw5x5_context(wb_arm.sets, K, stream) if world == 1 else None

    flops_all = sum_over_ranks(step_flops(wl), world, dev)
    bytes_all = sum_over_ranks(step_bytes(wl), world, dev)
    value = flops_all / (ms_step * 1e-3) / 1e12
    result = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic",
        "config": {
            "workload": workload_label(wl),
            "B": wl.B, "C_per_gpu": wl.C, "H": wl.H, "W": wl.W, "w": wl.w,
            "parallelism": "channel-sharded, %d rank(s), no collective" % world,
            "channels_of_rank0": list(channel_range(wl.C * world, world, 0)),
            "l2": "3 rotating input/output sets, %.0f MB per step > 126 MB L2"
                  % (step_bytes(wl) / 1e6),
            "timing": "CUDA graphs of 3 consecutive steps (one per buffer set) replayed, CUDA events, max over ranks",
        },
        "gbs": round(bytes_all / (ms_step * 1e-3) / 1e9, 1),
        "windows_channels_per_s": round(sum_over_ranks(wl.windows_per_channel * wl.C, world, dev)
                                        / (ms_step * 1e-3), 1),
        "kernels": kern,
        "gpu_launches": gpu_launches,
    }
    if wb_arm.fused:
        result["config"]["step"] = "fused cached forward + 3x3 (one launch)"
    # roofline of the dominant kernel (HBM-bound at w <= 14: AI ~ d/2 < ridge)
    dom = max(kern, key=lambda n: kern[n]["us"])
    ai = kernel_flops(wl, dom) / kernel_bytes(wl, dom)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    alu_tf = fp32_fma_peak_tflops(dev)
    if wl.dtype == "f32" and ai >= alu_tf * 1e12 / (peaks["hbm_gbs"] * 1e9):
        # fp32 runs on the CUDA cores: bound by their FMA rate
        result["roofline"] = {"bound": "alu", "kernel": dom, "achieved": kern[dom]["tflops"],
                              "peak": round(alu_tf, 1), "unit": "TFLOP/s",
                              "frac": round(kern[dom]["tflops"] / alu_tf, 4), "traffic": None,
                              "peak_source": "derived: SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz"}
    elif ai < ridge:
        result["roofline"] = {"bound": "hbm", "kernel": dom, "achieved": kern[dom]["gbs"],
                              "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": round(kern[dom]["gbs"] / peaks["hbm_gbs"], 4),
                              "traffic": recorded_traffic(dom) if wl.name == "train_bf16" else None,
                              "peak_source": peaks["source"]}
        if dom == "backward":
            result["roofline"]["launch"] = ("one backward call: the dX and dT kernels side by "
                                            "side on disjoint SMs; bytes x + dY + dX + T + dT")
    else:
        result["roofline"] = {"bound": "tensor", "kernel": dom, "achieved": kern[dom]["tflops"],
                              "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": round(kern[dom]["tflops"] / peaks["bf16_tflops"], 4),
                              "traffic": None, "peak_source": peaks["source"]}
    result["roofline"]["duration"] = ("average of K back-to-back calls of the entry point "
                                      "(CUDA events on the launching stream); kernels.*.us_isolated "
                                      "is one event pair around each call of the eager step")
    if alt:
        result["alternatives"] = alt
    top = alu_tf if wl.dtype == "f32" else peaks["bf16_tflops"]
    step_roof_tf = min(top, step_flops(wl) / step_bytes(wl) * peaks["hbm_gbs"] / 1e3)
    result["step_roofline_frac"] = round(value / world / step_roof_tf, 4)
    best_ms = pip_ms if pip_ms is not None else e2e_ms
    result["e2e"] = {"value": round(flops_all / (best_ms * 1e-3) / 1e12, 4), "unit": "TFLOP/s",
                     "ms_per_step": round(best_ms, 3), "h2d_bytes_per_step": h2d,
                     "d2h_bytes_per_step": d2h,
                     "copies": ("overlapped with the steps (2 buffer sets, copy-in and copy-out "
                                "streams)" if pip_ms is not None else "serial, on the step's stream"),
                     "ms_per_step_serial": round(e2e_ms, 3)}
    if context is not None:
        result["context_dw5x5"] = context
    if clk is not None:
        result["clocks"] = clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, wb_arm.host)
    gsteps.release()
    if world == 1 and not args.no_workloads:
        # the other workloads, each in its own graphs, with a clock record
        wclk = ClockSampler(local_rank)
        wclk.start()
        time.sleep(0.3)
        recs = time_workloads(dev, peaks, max(5, min(K, 20)))
        c = wclk.stop()
        result["workloads"] = {"steps_each": max(5, min(K, 20)), "records": recs}
        if c is not None:
            result["workloads"]["clocks"] = c
    return result


def run_reference(args, rank, world):
    """The oracle as it stands, on host cores, rank 0 only."""
    if rank != 0:
        return None
    import oracle
    wl = synth.WORKLOADS[WORKLOADS[args.workload]]
    bs = 8 if wl.kind == "train" else 4
    sub = wl.scaled(B=min(bs, wl.B))
    d = synth.draw(wl, seed=0)
    x, T = d["x"][:sub.B], d["T"]

    def one():
        if wl.kind == "train":
            dy = d["dY"][:sub.B]
            oracle.forward(x, T, wl.w)
            oracle.backward_dx(dy, T, wl.w)
            oracle.backward_dt(x, dy, wl.w)
        elif wl.kind == "cached_dw":
            y = oracle.forward_cached(x, oracle.expand(T, wl.w), wl.w)
            oracle.dw3x3(y, d["K"])
        elif wl.kind == "reparam":
            M = oracle.reparam_merge(T, d["Tk"], wl.w, synth.REPARAM_SMALL_WINDOW)
            oracle.forward_cached(x, M, wl.w)
        else:
            oracle.forward(x, T, wl.w)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    value = step_flops(sub) * args.steps / el / 1e12
    sample = "%d of %d images, all %d channels per step (fp64 C loops)" % (sub.B, wl.B, wl.C)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(wl), "sample": sample},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                         "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def spawn_ranks(n):
    """Starts one process per GPU (torch.distributed.run on this node, the
    rendezvous on 127.0.0.1) with the same arguments; returns its exit code."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", str(n), "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["wbmm", "reference"], default="wbmm")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="train")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads' timings after the headline step")
    ap.add_argument("--fused", action="store_true",
                    help="cached bf16 workloads: time the fused cached forward + 3x3 launch as "
                         "the step (the two calls become the alternatives)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "wbmm":
        ap.error("at least 3 warm-up steps")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")

    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        sys.exit(spawn_ranks(args.gpus))
    world = int(env_world or "1")
    if world != args.gpus:
        ap.error("--gpus %d but WORLD_SIZE=%d: launch one process per GPU "
                 "(torchrun --nproc-per-node %d), or omit WORLD_SIZE and let "
                 "bench.py start the ranks" % (args.gpus, world, args.gpus))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
