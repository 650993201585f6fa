"""Benchmark: BEVFormer-base Spatial Cross-Attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--value-dtype f32|bf16] [--rho coherent|uniform]

One step = one pass of the whole SCA forward over one synthetic batch: mask
compaction, the fused rebatched MSDA of all six cameras, the camera average
(sca_compact + sca_rebatched_forward + sca_camera_average, the same kernels
sca_forward launches).  Inputs are resident in HBM before timing; the L2 is
flushed (a 256 MiB write) before every step, outside the timed events.  Each
step is timed with CUDA events on the launching stream, per stage, and the
job time is the maximum over ranks of the summed step times.

N > 1 (torchrun, one process per GPU): every rank runs an independent replica
on its own seeded batch (weak scaling; the path has no exchange step).

Printed (rank 0): one JSON line with the metric, the roofline of the dominant
kernel (the rebatched gather) against the measured HBM copy bandwidth, the
oracle timed on the host as the CPU baseline, an end-to-end figure through
the one-call C ABI with host buffers, and the SM clocks seen during timing.

--impl reference times the oracle (plain C, double) on the host cores on the
same workload and metric, and prints the same kind of line with "impl":
"reference".
"""
import argparse
import hashlib
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MSDA sampled points/sec (G/s) + HBM GB/s fraction, BEVFormer-base SCA"
UNIT = "Gsamples/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = ("scale_deformable_attention_03_b200/csrc/msda_device.cuh",
                  "scale_deformable_attention_03_b200/csrc/sca.cu",
                  "scale_deformable_attention_03_b200/csrc/sca_gather_quad.cu")


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=("native", "reference"), default="native")
    p.add_argument("--value-dtype", choices=("f32", "bf16"), default="f32")
    p.add_argument("--rho", choices=("coherent", "uniform"), default="coherent")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--rows-iters", type=int, default=20,
                   help="timed calls per entry point in the next_rows section (0 = skip)")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="minimum host time of the oracle CPU baseline")
    return p.parse_args(argv)


# --------------------------------------------------------------------------
# helpers shared with the tests (no GPU needed)
# --------------------------------------------------------------------------

def rank_seed(rank):
    """Seed of a replica's synthetic batch: the workload's seed for rank 0,
    distinct seeds for the other ranks."""
    return 1003 + 1000 * rank


def workload_config(args):
    from scale_deformable_attention_03_b200 import inputs
    return {
        "workload": "bevformer-base-sca-forward",
        "B": 1, "Ncam": 6, "bev": "200x200", "Nq": 40000,
        "levels": [list(s) for s in inputs.SHAPES_BEVFORMER], "Nv_per_camera": 30825,
        "H": 8, "head_dim": 32, "P": 8, "R": 4,
        "value_dtype": args.value_dtype, "rho": args.rho,
        "mask": "1 + Bernoulli(0.5) cameras per query, non-zero anchor pattern",
        "l2": "flushed before every step (256 MiB write, outside the timed events)",
        "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU",
    }


def algorithmic_bytes(w, rows, hit_queries, value_elem):
    """Bytes each kernel / the whole step must move at least once.
    rows: rebatched rows (sum of count); hit_queries: queries seen by at
    least one camera."""
    S = w.H * w.L * w.P
    value = w.value.size * value_elem
    offsets_logits_per_query = S * 3 * 4
    ref_per_row = w.R * 2 * 4
    out_row = w.H * 32 * 4
    gather = (value + hit_queries * offsets_logits_per_query + rows * ref_per_row + rows * 4
              + rows * out_row)
    step = (value + w.B * w.Nq * offsets_logits_per_query + w.reference_points.nbytes
            + w.bev_mask.nbytes + w.B * w.Nq * out_row)
    return {"gather": int(gather), "step": int(step)}


def gather_kernel_name(w, bf16=False):
    """The rebatched-gather kernel sca_rebatched_forward launches here: the
    four-lane kernel for fp32 value and rows of up to 32 samples, else the
    table kernel (head pairs for bf16 value)."""
    if not bf16 and w.L * w.P <= 32:
        return "sca_gather_quad_kernel<float>"
    return "sca_gather_kernel<bf16, 1, 2>" if bf16 else "sca_gather_kernel<float>"


def aggregate(local_ms_total, local_samples, world):
    """Job time = max over ranks of the summed device time; work = sum."""
    if world == 1:
        return local_ms_total, local_samples
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([local_ms_total], dtype=torch.float64, device=dev)
    n = torch.tensor([float(local_samples)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), float(n.item())


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs, copy burst)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s pool measurement)"


def measured_bf16_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops)"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback (1.59 PFLOP/s pool measurement)"


def tsa_algorithmic_bytes(w, T, value_elem):
    """tsa_forward: every queue's value, offsets, logits and reference points
    once, the averaged output once."""
    S = w.H * w.L * w.P
    return int(w.value.size * value_elem + w.B * w.Nq * S * 3 * 4
               + w.B * w.Nq * w.R * 2 * 4 + (w.B // T) * w.Nq * w.H * 32 * 4)


def linear_algorithmic_bytes(M, N, K, y_elem, bias=True, residual=False):
    """msda_linear: x, w (and bias, residual) read once, y written once."""
    return int(M * K * 2 + N * K * 2 + (N * 4 if bias else 0) + (M * N * 4 if residual else 0)
               + M * N * y_elem)


def input_grads_algorithmic_bytes(w, rows):
    """sca_backward_inputs: logits, positions, the rebatched gradients of the
    seen rows once; the three gradients written once."""
    S = w.H * w.L * w.P
    return int(w.B * w.Nq * S * 4 + w.B * w.Ncam * w.Nq * 4 + rows * S * 3 * 4
               + w.B * w.Nq * S * 3 * 4 + w.Ncam * w.B * w.Nq * w.R * 2 * 4)


def sca_backward_algorithmic_bytes(w, rows, hit_queries, value_elem):
    """sca_backward: the forward's inputs once (value, offsets and logits of
    seen queries, reference points, mask), grad_out once, grad_value written
    once (the atomics' read-modify-write is not counted), the rebatched
    location and weight gradients of the seen rows written once."""
    S = w.H * w.L * w.P
    return int(w.value.size * value_elem + hit_queries * S * 3 * 4 + rows * w.R * 2 * 4
               + w.bev_mask.nbytes + w.B * w.Nq * w.H * 32 * 4 + w.value.size * 4
               + rows * S * 3 * 4)


def kernel_source_digest():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(value_dtype):
    """DRAM bytes per gather launch from the committed ncu record
    (profiles/traffic.json), when it was taken on the current kernel sources;
    None otherwise."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_sources_sha256_16") != kernel_source_digest():
        return None
    v = rec.get("dram_bytes_per_launch", {}).get(value_dtype)
    return int(v) if v is not None else None


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every few
    milliseconds while the timed region runs (a background thread)."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device):
        import threading
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.stop_flag = threading.Event()
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = self._handle(torch_device)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle,
                                                                  pynvml.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None

    def _handle(self, dev):
        import torch
        pynvml = self.nvml
        p = torch.cuda.get_device_properties(dev)
        try:
            bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(dev)

    def _run(self):
        pynvml = self.nvml
        get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(self.handle,
                                                                        pynvml.NVML_CLOCK_SM)))
                bits = get_reasons(self.handle)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            self.stop_flag.wait(0.005)

    def start(self):
        if self.nvml is None:
            return
        import threading
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag.set()
        self.thread.join()
        if not self.samples:
            return None
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "NVML, every 5 ms during the timed steps"}


# --------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, one host core
# --------------------------------------------------------------------------

def oracle_step(w, q0, q1, value64=None):
    """One oracle SCA forward over BEV queries q0 .. q1 - 1 of the workload
    (all cameras, full value maps). Returns sampled points."""
    import oracle
    q = slice(q0, q1)
    out = oracle.sca_forward(w.value if value64 is None else value64, w.spatial_shapes,
                             w.level_start_index,
                             np.ascontiguousarray(w.reference_points[:, :, q]),
                             np.ascontiguousarray(w.bev_mask[:, :, q]),
                             np.ascontiguousarray(w.sampling_offsets[:, q]),
                             np.ascontiguousarray(w.attention_logits[:, q]))
    assert out.shape[1] == q1 - q0
    rows = int(np.count_nonzero(w.bev_mask[:, :, q].any(-1)))
    return rows * w.H * w.L * w.P


def cpu_baseline(w, min_seconds):
    """The oracle as it stands on the host cores: full workload passes on one
    core, then passes split into query slices over every core (threads: the
    C oracle runs without the Python lock).  The value map is widened to
    double once, outside the timed passes (the oracle's input type)."""
    import concurrent.futures as cf
    import oracle
    oracle.lib()
    v64 = np.ascontiguousarray(w.value, dtype=np.float64)
    done, samples, t0 = 0, 0, time.perf_counter()
    while True:
        samples += oracle_step(w, 0, w.Nq, v64)
        done += 1
        el1 = time.perf_counter() - t0
        if el1 >= min_seconds:
            break
    one = samples / el1 / 1e9
    cores = os.cpu_count() or 1
    step = max(200, (w.Nq // (4 * cores)) // 200 * 200)  # whole BEV rows per slice
    slices = [(q, min(w.Nq, q + step)) for q in range(0, w.Nq, step)]
    done_m, samples_m = 0, 0
    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        t0 = time.perf_counter()
        while True:
            samples_m += sum(ex.map(lambda s: oracle_step(w, s[0], s[1], v64), slices))
            done_m += 1
            elm = time.perf_counter() - t0
            if elm >= min_seconds / 2:
                break
    many = samples_m / elm / 1e9
    return {"value": many, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{done_m} full workload pass(es) of the C oracle (double) split into "
                      f"{len(slices)} query slices over {cores} threads, {elm:.1f} s",
            "single_core": {"value": one, "unit": UNIT, "cores": 1,
                            "sample": f"{done} full workload pass(es) on one core, {el1:.1f} s"}}


def run_reference(args):
    """The oracle as it stands on the machine's host cores (threads over query
    slices; the C oracle runs without the Python lock), one step = one SCA
    forward over a bounded, whole-BEV-row sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import concurrent.futures as cf

    from scale_deformable_attention_03_b200 import inputs
    from oracle import build as oracle_build
    import oracle
    oracle_build.build()
    oracle.lib()
    w = inputs.workload3(seed=rank_seed(0), value_dtype=args.value_dtype, rho=args.rho)
    v64 = np.ascontiguousarray(w.value, dtype=np.float64)
    cores = os.cpu_count() or 1

    def step(nq, ex):
        per = max(200, (nq // (4 * cores)) // 200 * 200)  # whole BEV rows per slice
        slices = [(q, min(nq, q + per)) for q in range(0, nq, per)]
        return sum(ex.map(lambda s: oracle_step(w, s[0], s[1], v64), slices))

    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        t0 = time.perf_counter()
        step(w.Nq, ex)
        t_full = time.perf_counter() - t0
        budget = 150.0  # seconds for warm-up + timed steps
        frac = min(1.0, budget / max(1e-9, (args.steps + args.warmup) * t_full))
        nq = max(200, int(w.Nq * frac) // 200 * 200)  # whole BEV rows of 200 cells
        for _ in range(args.warmup):
            step(nq, ex)
        samples, t0 = 0, time.perf_counter()
        for _ in range(args.steps):
            samples += step(nq, ex)
        el = time.perf_counter() - t0
    value = samples / el / 1e9
    sample = (f"first {nq} of {w.Nq} BEV queries per step (all 6 cameras, full value maps), "
              f"C oracle in double over {cores} host threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# native arm
# --------------------------------------------------------------------------

def measure_replica(args, rank, world, barrier):
    """The device section of one replica: the timed SCA forward steps, the
    warm-L2 gather, the end-to-end leg through sca_forward with host buffers
    and (one GPU) the further entry points.  barrier() is called at the same
    points on every rank.  Returns this rank's local results."""
    import torch

    import scale_deformable_attention_03_b200 as msda
    from scale_deformable_attention_03_b200 import inputs

    msda.lib()  # fail loudly before any work when the library is missing
    stream = torch.cuda.current_stream()

    w = inputs.workload3(seed=rank_seed(rank), value_dtype=args.value_dtype, rho=args.rho)
    bf16 = args.value_dtype == "bf16"

    def d(a):
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    value = d(w.value_bf16.view(np.int16)).view(torch.bfloat16) if bf16 else d(w.value)
    ref, mask = d(w.reference_points), d(w.bev_mask)
    off, logits = d(w.sampling_offsets), d(w.attention_logits)
    shapes, starts = w.spatial_shapes, w.level_start_index
    dims = msda.Dims(w.B, w.Ncam, w.Nq, w.Nv, w.H, w.L, w.P, w.R)
    cws = torch.empty(max(16, msda.sca_compact_workspace_size(dims)), dtype=torch.uint8,
                      device="cuda")
    idx = torch.empty((w.B, w.Ncam, w.Nq), dtype=torch.int32, device="cuda")
    count = torch.empty((w.B, w.Ncam), dtype=torch.int32, device="cuda")
    pos = torch.empty_like(idx)
    hits = torch.empty((w.B, w.Nq), dtype=torch.int32, device="cuda")
    out_rb = torch.empty((w.B, w.Ncam, w.Nq, w.H * 32), dtype=torch.float32, device="cuda")
    out = torch.empty((w.B, w.Nq, w.H * 32), dtype=torch.float32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    L = msda.lib()
    i64 = msda._i64p
    vdt = msda.MSDA_BF16 if bf16 else msda.MSDA_F32
    sp, st = shapes.ctypes.data_as(i64), starts.ctypes.data_as(i64)
    P = msda._ptr
    sptr = msda._stream(stream)

    def compact():
        msda._check(L.sca_compact(P(mask), dims, P(cws), cws.numel(), P(idx), P(count), P(pos),
                                  P(hits), sptr), "sca_compact")

    def gather():
        msda._check(L.sca_rebatched_forward(P(value), vdt, sp, st, P(ref), P(off), P(logits),
                                            P(idx), P(count), dims, P(out_rb), sptr),
                    "sca_rebatched_forward")

    def average():
        msda._check(L.sca_camera_average(P(out_rb), P(pos), P(hits), dims, P(out), sptr),
                    "sca_camera_average")

    fws = torch.empty(msda.msda_workspace_size(dims), dtype=torch.uint8, device="cuda")

    def forward():  # the step as a user runs it: the same kernels in one call
        msda._check(L.sca_forward(P(value), vdt, sp, st, P(ref), P(mask), P(off), P(logits),
                                  dims, P(fws), fws.numel(), P(out), sptr), "sca_forward")

    # compaction (count, scatter; a scan pass between them above 64 chunks of
    # 1024 queries), the gather, the average
    launches_per_step = 4 if (w.Nq + 1023) // 1024 <= 64 else 5
    compact()
    torch.cuda.synchronize()
    rows = int(count.sum().item())
    hit_queries = int((hits > 0).sum().item())
    samples_per_step = rows * w.H * w.L * w.P
    nbytes = algorithmic_bytes(w, rows, hit_queries, 2 if bf16 else 4)

    for _ in range(args.warmup):
        flush.zero_()
        forward()
    torch.cuda.synchronize()

    # The timed steps: one sca_forward call each, events only around it, so
    # that its kernels overlap at their boundaries as in any use (the scatter
    # pass, the gather and the average are programmatic dependent launches).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    # The same kernels as three calls with events between the stages, for the
    # per-kernel times (the gather's feeds the roofline); an event between two
    # kernels ends their overlap, so these stages add up to a little more.
    stage_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
                 for _ in range(args.steps)]
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for e in evs:
        flush.zero_()
        e[0].record(stream)
        forward()
        e[1].record(stream)
    for e in stage_evs:
        flush.zero_()
        e[0].record(stream)
        compact()
        e[1].record(stream)
        gather()
        e[2].record(stream)
        average()
        e[3].record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    # the gather again with a warm L2 (no flush between launches), for reference
    warm_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(min(args.steps, 50))]
    for a, b in warm_evs:
        a.record(stream)
        gather()
        b.record(stream)
    torch.cuda.synchronize()
    warm_gather_ms = float(np.median([a.elapsed_time(b) for a, b in warm_evs]))
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    staged_ms = [e[0].elapsed_time(e[3]) for e in stage_evs]
    gather_ms = [e[1].elapsed_time(e[2]) for e in stage_evs]
    compact_ms = [e[0].elapsed_time(e[1]) for e in stage_evs]
    avg_ms = [e[2].elapsed_time(e[3]) for e in stage_evs]
    # ---- end to end through the one-call C ABI, host buffers ----
    # Every step copies its inputs from pinned host memory, runs sca_forward
    # and copies its result back.  Two device buffer sets let the copies of
    # step i + 1 (copy stream) overlap the kernels of step i (compute stream)
    # and the read-back of step i - 1 (read-back stream).
    host = {k: torch.from_numpy(np.ascontiguousarray(a)).pin_memory() for k, a in (
        ("value", w.value_bf16.view(np.int16) if bf16 else w.value),
        ("ref", w.reference_points), ("mask", w.bev_mask), ("off", w.sampling_offsets),
        ("logits", w.attention_logits))}
    host_out = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    ws = torch.empty(msda.msda_workspace_size(dims), dtype=torch.uint8, device="cuda")
    dev_in = [{k: torch.empty(v.shape, dtype=v.dtype, device="cuda") for k, v in host.items()}
              for _ in range(2)]
    dev_out = [torch.empty_like(out) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = host_out[0].numel() * 4
    copy_s, back_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    computed = [ev(), ev()]
    read_back = [ev(), ev()]

    def e2e_step(i):
        j = i % 2
        copied = ev()
        with torch.cuda.stream(copy_s):
            copy_s.wait_event(computed[j])   # step i - 2 has finished reading set j
            for k in host:
                dev_in[j][k].copy_(host[k], non_blocking=True)
            copied.record(copy_s)
        stream.wait_event(copied)
        stream.wait_event(read_back[j])      # step i - 2's result has left dev_out[j]
        d_in = dev_in[j]
        v = d_in["value"].view(torch.bfloat16) if bf16 else d_in["value"]
        msda._check(L.sca_forward(P(v), vdt, sp, st, P(d_in["ref"]), P(d_in["mask"]),
                                  P(d_in["off"]), P(d_in["logits"]), dims, P(ws), ws.numel(),
                                  P(dev_out[j]), sptr), "sca_forward")
        computed[j].record(stream)
        with torch.cuda.stream(back_s):
            back_s.wait_event(computed[j])
            host_out[j].copy_(dev_out[j], non_blocking=True)
            read_back[j].record(back_s)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_s.wait_event(e0)
    for i in range(args.e2e_steps):
        e2e_step(i)
    stream.wait_stream(back_s)
    stream.wait_stream(copy_s)
    e1.record(stream)
    torch.cuda.synchronize()
    res = {"w": w, "bf16": bf16, "step_ms": step_ms, "staged_ms": staged_ms,
           "gather_ms": gather_ms,
           "compact_ms": compact_ms, "avg_ms": avg_ms, "warm_gather_ms": warm_gather_ms,
           "samples_per_step": samples_per_step, "rows": rows, "nbytes": nbytes,
           "e2e_ms": e0.elapsed_time(e1), "h2d": int(h2d), "d2h": int(d2h), "clocks": clocks,
           "launches_per_step": launches_per_step}
    if world == 1 and args.rows_iters > 0:
        tensors = {"value": value, "ref": ref, "mask": mask, "off": off, "logits": logits,
                   "step_bytes": nbytes["step"], "samples": samples_per_step}
        peak, _ = measured_hbm_peak()
        res["next_rows"] = measure_next_rows(args, w, tensors, flush, stream, peak)
    return res


def run_native(args, backend="nccl", replica=measure_replica):
    """One replica per rank (weak scaling): the device section (`replica`),
    then the job time (max over ranks of the summed step times) and work (sum
    over ranks) through the process group; rank 0 prints the JSON line."""
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if backend == "nccl":
        import torch
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        kw = {}
        if backend == "nccl":
            import torch
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)

    def barrier():
        if world > 1:
            dist.barrier()

    res = replica(args, rank, world, barrier)
    step_ms = res["step_ms"]
    total_ms, total_samples = aggregate(sum(step_ms), res["samples_per_step"] * args.steps, world)
    value_gs = total_samples / (total_ms * 1e-3) / 1e9
    e2e_ms, e2e_samples = aggregate(res["e2e_ms"], res["samples_per_step"] * args.e2e_steps, world)
    e2e_gs = e2e_samples / (e2e_ms * 1e-3) / 1e9
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    w, nbytes = res["w"], res["nbytes"]
    gather_ms, compact_ms, avg_ms = res["gather_ms"], res["compact_ms"], res["avg_ms"]
    warm_gather_ms, samples_per_step = res["warm_gather_ms"], res["samples_per_step"]
    rows, h2d, d2h, clocks = res["rows"], res["h2d"], res["d2h"], res["clocks"]
    launches_per_step = res["launches_per_step"]
    peak, peak_src = measured_hbm_peak()
    g_ms = float(np.mean(gather_ms))
    # the step's algorithmic bytes (value once, every query's offsets and
    # logits, reference points, mask, output once) over the dominant kernel's
    # time; the gather's own bytes (with its rebatched rows) beside it
    achieved = nbytes["step"] / (g_ms * 1e-3) / 1e9
    achieved_own = nbytes["gather"] / (g_ms * 1e-3) / 1e9
    traffic = recorded_traffic(args.value_dtype)
    step_mean = float(np.mean(step_ms))
    line = {
        "metric": METRIC, "value": value_gs, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config(args),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": gather_kernel_name(w, res["bf16"]), "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": nbytes["step"],
                     "algorithmic_bytes_note": "the step's bytes (value, offsets and logits "
                                               "of every query, reference points, mask, "
                                               "output), each once",
                     "gather_own_bytes_per_launch": nbytes["gather"],
                     "gather_own_frac": achieved_own / peak,
                     "launch_ms": g_ms},
        "step": {"algorithmic_bytes": nbytes["step"],
                 "hbm_gbs": nbytes["step"] / (step_mean * 1e-3) / 1e9,
                 "hbm_frac": nbytes["step"] / (step_mean * 1e-3) / 1e9 / peak,
                 "ms": {"compact": float(np.mean(compact_ms)), "gather": g_ms,
                        "average": float(np.mean(avg_ms)), "step": step_mean,
                        "staged_step": float(np.mean(res["staged_ms"]))},
                 "timing": "step: one sca_forward call per step, events around it; "
                           "compact / gather / average: the same kernels as three calls "
                           "with events between them, in a second pass of as many steps",
                 "step_ms_percentiles": {"p10": float(np.percentile(step_ms, 10)),
                                         "median": float(np.median(step_ms)),
                                         "p90": float(np.percentile(step_ms, 90))},
                 "gather_ms_warm_l2_median": warm_gather_ms,
                 "samples": samples_per_step, "rebatched_rows": rows},
        "e2e": {"value": e2e_gs, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "api": "sca_forward (one call)",
                "steps": args.e2e_steps,
                "pipelining": "copies of step i+1 and read-back of step i-1 overlap the "
                              "kernels of step i (two buffer sets, three streams)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if "next_rows" in res:
        line["next_rows"] = res["next_rows"]
    if world == 1 and args.cpu_seconds > 0:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(line), flush=True)
    return 0




# --------------------------------------------------------------------------
# the other entry points of the path, each on its full workload
# --------------------------------------------------------------------------

def measure_next_rows(args, w, tensors, flush, stream, hbm_peak):
    """Mean CUDA-event time of each further entry point (after three warm-up
    calls, the L2 flushed before every call, outside the events), with its
    algorithmic bytes against the measured HBM copy bandwidth."""
    import torch

    import scale_deformable_attention_03_b200 as msda
    from scale_deformable_attention_03_b200 import inputs

    iters = args.rows_iters

    def timed(fn, n=iters):
        for _ in range(3):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in evs]))

    def hbm(nbytes, ms):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": ms, "algorithmic_bytes": int(nbytes), "achieved_gbs": gbs,
                "hbm_frac": gbs / hbm_peak}

    rows = {}
    bf16 = args.value_dtype == "bf16"
    with_cpu = args.cpu_seconds > 0

    def cpu_rate(call, work, unit, what):
        """The oracle timed on one host core on a bounded slice of the same
        workload (one call), as work per second."""
        t0 = time.perf_counter()
        call()
        el = time.perf_counter() - t0
        return {"value": work / el, "unit": unit, "cores": 1, "kind": "oracle",
                "sample": f"{what}: {el:.2f} s on one host core"}
    value, ref, mask, off, logits = (tensors[k] for k in ("value", "ref", "mask", "off",
                                                          "logits"))
    shapes, starts = w.spatial_shapes, w.level_start_index

    # f2: query-major SCA forward (one kernel, the whole step's algorithmic bytes)
    out = torch.empty((w.B, w.Nq, w.H * 32), dtype=torch.float32, device="cuda")
    ms = timed(lambda: msda.sca_forward_query_major(value, shapes, starts, ref, mask, off,
                                                    logits, out=out))
    r = hbm(tensors["step_bytes"], ms)
    r.update(kernel="sca_query_major_kernel", workload="bevformer-base-sca-forward",
             gsamples_per_s=tensors["samples"] / (ms * 1e-3) / 1e9)
    rows["sca_forward_query_major"] = r

    # the same SCA forward with bf16 value (BEVFormer-base's bf16 variant):
    # sca_forward (compaction, head-pair gather, camera average) and the
    # query-major kernel
    if not bf16:
        vb16 = value.to(torch.bfloat16)  # round to nearest even, as the inputs module does
        step_b16 = tensors["step_bytes"] - w.value.size * 2
        dims16 = msda.Dims(w.B, w.Ncam, w.Nq, w.Nv, w.H, w.L, w.P, w.R)
        ws16 = torch.empty(msda.msda_workspace_size(dims16), dtype=torch.uint8, device="cuda")
        ms = timed(lambda: msda.sca_forward(vb16, shapes, starts, ref, mask, off, logits,
                                            out=out, workspace=ws16))
        r = hbm(step_b16, ms)
        r.update(kernel="sca_count + sca_scatter + "
                        f"{gather_kernel_name(w, True)} + sca_average (sca_forward's bf16 path)",
                 workload="bevformer-base-sca-forward, bf16 value",
                 gsamples_per_s=tensors["samples"] / (ms * 1e-3) / 1e9)
        rows["sca_forward_bf16"] = r
        ms = timed(lambda: msda.sca_forward_query_major(vb16, shapes, starts, ref, mask, off,
                                                        logits, out=out))
        r = hbm(step_b16, ms)
        r.update(kernel="sca_query_major_kernel<bf16, 1, 2>",
                 workload="bevformer-base-sca-forward, bf16 value",
                 gsamples_per_s=tensors["samples"] / (ms * 1e-3) / 1e9)
        rows["sca_forward_query_major_bf16"] = r
        del vb16, ws16

    # the tiny single-level MSDA (16 x 16 map, 256 queries, two heads): given
    # locations and host-softmaxed weights; launch-latency bound, so the time
    # (not a bandwidth fraction) is the figure
    wk = inputs.workload1()
    a = wk.attention_logits.astype(np.float64)
    wts1 = np.exp(a - a.max(-1, keepdims=True))
    wts1 = (wts1 / wts1.sum(-1, keepdims=True)).astype(np.float32)
    v1, l1, w1 = (torch.from_numpy(np.ascontiguousarray(x)).cuda()
                  for x in (wk.value, wk.sampling_locations, wts1))
    o1 = torch.empty((wk.B, wk.Nq, wk.H * 32), dtype=torch.float32, device="cuda")
    ms = timed(lambda: msda.msda_forward(v1, wk.spatial_shapes, wk.level_start_index, l1, w1,
                                         out=o1))
    S1 = wk.H * wk.L * wk.P
    r = {"ms": ms, "us": ms * 1e3, "workload": wk.name, "samples": wk.B * wk.Nq * S1,
         "kernel": "msda_forward_group_kernel (rows of L·P <= 16)",
         "note": "0.15 MB of algorithmic bytes: bound by launch latency, not by memory"}
    if with_cpu:
        import oracle
        r["cpu_oracle"] = cpu_rate(
            lambda: oracle.msda_forward(wk.value, wk.spatial_shapes, wk.level_start_index,
                                        wk.sampling_locations, wts1),
            wk.B * wk.Nq * S1 / 1e9, UNIT, "the whole workload")
    rows["msda_forward_tiny"] = r
    del v1, l1, w1, o1

    # the plain fused MSDA: the Deformable-DETR encoder and the TSA queues as a batch
    for name, wk, kname in (
            ("msda_forward_fused_detr", inputs.workload2(), "msda_forward_group_kernel<float, true, 4>"),
            ("msda_forward_fused_tsa_batch2", inputs.workload4(),
             "msda_forward_group_kernel<float, true, 2>")):
        dv = {k: torch.from_numpy(np.ascontiguousarray(a)).cuda() for k, a in (
            ("value", wk.value), ("ref", wk.reference_points), ("off", wk.sampling_offsets),
            ("logits", wk.attention_logits))}
        o = torch.empty((wk.B, wk.Nq, wk.H * 32), dtype=torch.float32, device="cuda")
        fa = (dv["value"], wk.spatial_shapes, wk.level_start_index, dv["ref"], dv["off"],
              dv["logits"])
        ms = timed(lambda: msda.msda_forward_fused(*fa, out=o))
        S = wk.H * wk.L * wk.P
        nbytes = (wk.value.nbytes + wk.B * wk.Nq * S * 12 + wk.reference_points.nbytes
                  + o.numel() * 4)
        r = hbm(nbytes, ms)
        r.update(kernel=kname, workload=wk.name,
                 gsamples_per_s=wk.B * wk.Nq * S / (ms * 1e-3) / 1e9)
        if with_cpu:
            import oracle
            nq = wk.Nq
            sl = (slice(None), slice(0, nq))
            r["cpu_oracle"] = cpu_rate(
                lambda: oracle.msda_forward_fused(
                    wk.value, wk.spatial_shapes, wk.level_start_index,
                    np.ascontiguousarray(wk.reference_points[sl]),
                    np.ascontiguousarray(wk.sampling_offsets[sl]),
                    np.ascontiguousarray(wk.attention_logits[sl])),
                wk.B * nq * S / 1e9, UNIT, f"all {nq} queries")
        rows[name] = r
        if name == "msda_forward_fused_detr":
            # the same encoder's backward from given locations and weights
            # (prepared with plain torch ops, outside the timed region)
            wh = torch.tensor([[w_, h_] for h_, w_ in wk.spatial_shapes], dtype=torch.float32,
                              device="cuda").view(1, 1, 1, wk.L, 1, 2)
            loc = (dv["ref"].view(wk.B, wk.Nq, 1, 1, 1, 2) + dv["off"] / wh).contiguous()
            wts = torch.softmax(dv["logits"].view(wk.B, wk.Nq, wk.H, -1), -1).view(
                dv["logits"].shape).contiguous()
            gout = torch.randn((wk.B, wk.Nq, wk.H * 32), device="cuda")
            grads = msda.msda_backward(dv["value"], wk.spatial_shapes, wk.level_start_index,
                                       loc, wts, gout)
            ms = timed(lambda: msda.msda_backward(dv["value"], wk.spatial_shapes,
                                                  wk.level_start_index, loc, wts, gout, *grads))
            # value read and grad_value written once, locations and weights
            # read and their gradients written once, grad_out read once
            r = hbm(2 * wk.value.nbytes + wk.B * wk.Nq * S * 12 * 2 + gout.numel() * 4, ms)
            r.update(kernel="zero_kernel + backward_group_kernel<float, 4, false, false>",
                     workload=wk.name, gsamples_per_s=wk.B * wk.Nq * S / (ms * 1e-3) / 1e9)
            rows["msda_backward_detr"] = r
            del loc, wts, gout, grads
        del dv, o, fa

    # f4: TSA, two queues of the 200x200 BEV, ego motion (1.7 m, -0.9 m, 4 deg)
    w4 = inputs.workload4()
    ego = torch.tensor([[[1.7, -0.9, 4.0], [0.0, 0.0, 0.0]]], dtype=torch.float32,
                       device="cuda")
    ref4 = msda.tsa_reference_points(ego, 200, 200)
    v4 = torch.from_numpy(w4.value).cuda()
    off4 = torch.from_numpy(w4.sampling_offsets).cuda()
    lg4 = torch.from_numpy(w4.attention_logits).cuda()
    out4 = torch.empty((1, w4.Nq, w4.H * 32), dtype=torch.float32, device="cuda")
    ref4v = ref4.view(2, w4.Nq, 1, 2)
    ms = timed(lambda: msda.tsa_forward(v4, w4.spatial_shapes, w4.level_start_index, ref4v,
                                        off4, lg4, 2, out=out4))
    r = hbm(tsa_algorithmic_bytes(w4, 2, 4), ms)
    r.update(kernel="tsa_forward_group_kernel<float, 2, 2>",
             workload="bevformer-tsa 2 queues x 200x200, H=8, P=4, fp32",
             gsamples_per_s=2 * w4.Nq * w4.H * w4.L * w4.P / (ms * 1e-3) / 1e9)
    nq4 = 20000
    sl4 = (slice(None), slice(0, nq4))
    if with_cpu:
        import oracle
        ref4_np = oracle.tsa_reference_points(
            200, 200, np.array([[[1.7, -0.9, 4.0], [0.0, 0.0, 0.0]]])).reshape(2, -1, 1, 2)
        r["cpu_oracle"] = cpu_rate(
            lambda: oracle.tsa_forward(w4.value, w4.spatial_shapes, w4.level_start_index,
                                       np.ascontiguousarray(ref4_np[sl4]),
                                       np.ascontiguousarray(w4.sampling_offsets[sl4]),
                                       np.ascontiguousarray(w4.attention_logits[sl4]), 2),
            2 * nq4 * w4.H * w4.L * w4.P / 1e9, UNIT, f"the first {nq4} BEV queries")
    rows["tsa_forward"] = r
    ms = timed(lambda: msda.tsa_reference_points(ego, 200, 200, out=ref4))
    rows["tsa_reference_points"] = hbm(2 * w4.Nq * 8 + 24, ms)
    go4 = torch.randn((1, w4.Nq, w4.H * 32), device="cuda")
    tws = torch.empty(int(msda.lib().tsa_backward_workspace_size(
        msda.Dims(1, 1, w4.Nq, w4.Nv, w4.H, w4.L, w4.P, w4.R), 2)), dtype=torch.uint8,
        device="cuda")
    ms = timed(lambda: msda.tsa_backward(v4, w4.spatial_shapes, w4.level_start_index, ref4v,
                                         off4, lg4, 2, go4, workspace=tws))
    S4 = w4.H * w4.L * w4.P
    r = hbm(tsa_algorithmic_bytes(w4, 2, 4) + w4.Nq * w4.H * 32 * 4 + w4.value.size * 4
            + 2 * w4.Nq * (S4 * 3 + w4.R * 2) * 4, ms)
    r.update(kernel="zero_kernel + backward_group_kernel<float, 2, true, false> + "
                    "sca_offset_logit_grads_group_kernel<2, true>",
             workload="bevformer-tsa 2 queues x 200x200, H=8, P=4, fp32",
             gsamples_per_s=2 * w4.Nq * S4 / (ms * 1e-3) / 1e9)
    if with_cpu:
        go4_np = np.random.Generator(np.random.PCG64(4)).standard_normal((1, nq4, w4.H * 32))
        r["cpu_oracle"] = cpu_rate(
            lambda: oracle.tsa_backward(w4.value, w4.spatial_shapes, w4.level_start_index,
                                        np.ascontiguousarray(ref4_np[sl4]),
                                        np.ascontiguousarray(w4.sampling_offsets[sl4]),
                                        np.ascontiguousarray(w4.attention_logits[sl4]), 2,
                                        go4_np),
            2 * nq4 * S4 / 1e9, UNIT, f"the first {nq4} BEV queries")
    rows["tsa_backward"] = r
    del v4, off4, lg4, out4, ref4, go4, tws

    # A12: the value projection of all six cameras' features, M = 6 * 30825
    g = torch.Generator(device="cuda").manual_seed(7)
    M, N, K = w.Ncam * w.Nv, 256, 256
    x = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
    wt = (torch.randn((N, K), device="cuda", generator=g) / 16).to(torch.bfloat16)
    bias = torch.randn(N, device="cuda", generator=g)
    peak_tf, peak_tf_src = measured_bf16_peak()
    for y_dtype, y_elem in (("f32", 4), ("bf16", 2)):
        y = torch.empty((M, N), device="cuda",
                        dtype=torch.float32 if y_dtype == "f32" else torch.bfloat16)
        ms = timed(lambda: msda.msda_linear(x, wt, bias, out=y))
        r = hbm(linear_algorithmic_bytes(M, N, K, y_elem), ms)
        tflops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        r.update(kernel="proj_gemm_kernel (tcgen05)", shape=[M, N, K], y_dtype=y_dtype,
                 tflops=tflops, tensor_frac=tflops / peak_tf, tensor_peak_source=peak_tf_src)
        if with_cpu and y_dtype == "f32":
            import oracle
            mc = 10000
            xs = x[:mc].float().cpu().numpy()
            wts = wt.float().cpu().numpy()
            r["cpu_oracle"] = cpu_rate(lambda: oracle.linear(xs, wts),
                                       2.0 * mc * N * K / 1e12, "TFLOP/s",
                                       f"{mc} rows of the same projection")
        rows[f"msda_linear_value_proj_{y_dtype}"] = r
    del x, y

    # f1: the whole SCA module forward (projections + SCA + output projection)
    C = w.H * 32
    S = w.H * w.L * w.P
    q = torch.randn((w.B, w.Nq, C), device="cuda", generator=g)
    feats = torch.randn((w.B, w.Ncam, w.Nv, C), device="cuda", generator=g).to(torch.bfloat16)

    def lin(n_out):
        return ((torch.randn((n_out, C), device="cuda", generator=g) / 16).to(torch.bfloat16),
                torch.randn(n_out, device="cuda", generator=g) * 0.1)

    (wv, bv), (wo_, bo_), (wa, ba), (wout, bout) = lin(C), lin(2 * S), lin(S), lin(C)
    mod_out = torch.empty_like(q)
    vdt = torch.bfloat16 if bf16 else None
    mod_dims = msda.Dims(w.B, w.Ncam, w.Nq, w.Nv, w.H, w.L, w.P, w.R)
    mod_ws = torch.empty(int(msda.lib().sca_module_workspace_size(
        mod_dims, msda.MSDA_BF16 if bf16 else msda.MSDA_F32)), dtype=torch.uint8, device="cuda")
    ms = timed(lambda: msda.sca_module_forward(q, None, feats, wv, bv, wo_, bo_, wa, ba, wout,
                                               bout, ref, mask, shapes, starts, w.L, w.P,
                                               value_dtype=vdt, out=mod_out,
                                               workspace=mod_ws))
    rows["sca_module_forward"] = {"ms": ms, "workload": "bevformer-base SCA module, C=256",
                                  "gsamples_per_s": tensors["samples"] / (ms * 1e-3) / 1e9}
    del feats, mod_out, mod_ws

    # f1: the camera average fused into the output projection (the module's
    # last step for fp32 value)
    if not bf16:
        idx, cnt, pos, hits = msda.sca_compact(mask)
        rb = msda.sca_rebatched_forward(value, shapes, starts, ref, off, logits, idx, cnt)
        n_rows = int(cnt.sum().item())
        resid = q.reshape(w.B * w.Nq, C)
        y = torch.empty_like(resid)
        ms = timed(lambda: msda.sca_camera_average_linear(rb, pos, hits, wout, bout, resid, out=y))
        nbytes = (n_rows * C * 4 + w.B * w.Ncam * w.Nq * 4 + w.B * w.Nq * 4 + C * C * 2 + C * 4
                  + 2 * w.B * w.Nq * C * 4)
        r = hbm(nbytes, ms)
        r.update(kernel="proj_gemm_kernel<averaged X> (tcgen05)",
                 workload="bevformer-base output projection, C=256, residual",
                 algorithmic_bytes_note="the rebatched rows once, pos, hits, W_o, b_o, residual, y")
        rows["sca_camera_average_linear"] = r
        del rb, y, resid
    del q

    # f3: gradients of offsets, logits and reference points from the rebatched ones
    idx, cnt, pos, hits = msda.sca_compact(mask)
    gout = torch.randn((w.B, w.Nq, C), device="cuda", generator=g)
    _, gl, gw = msda.sca_rebatched_backward(value, shapes, starts, ref, off, logits, gout, idx,
                                            cnt, hits)
    n_rows = int(cnt.sum().item())
    bufs = msda.sca_backward_inputs(shapes, starts, logits, pos, gl, gw, w.Ncam, w.R)
    ms = timed(lambda: msda.sca_backward_inputs(shapes, starts, logits, pos, gl, gw, w.Ncam,
                                                w.R, out=bufs))
    r = hbm(input_grads_algorithmic_bytes(w, n_rows), ms)
    r.update(kernel="sca_offset_logit_grads_kernel<1, true> (reference points fused)")
    rows["sca_backward_inputs"] = r
    del gl, gw, bufs, gout

    # A10/A11: the SCA backward of the training-step shape (B = 2, bf16 value)
    w5 = inputs.workload5()
    d5 = {k: torch.from_numpy(np.ascontiguousarray(a)).cuda() for k, a in (
        ("ref", w5.reference_points), ("mask", w5.bev_mask), ("off", w5.sampling_offsets),
        ("logits", w5.attention_logits), ("gout", w5.grad_out))}
    v5 = torch.from_numpy(w5.value_bf16.view(np.int16)).cuda().view(torch.bfloat16)
    args5 = (v5, w5.spatial_shapes, w5.level_start_index, d5["ref"], d5["mask"], d5["off"],
             d5["logits"], d5["gout"])
    g5 = msda.sca_backward(*args5)
    _, cnt5, _, hits5 = msda.sca_compact(d5["mask"])
    rows5, hitq5 = int(cnt5.sum().item()), int((hits5 > 0).sum().item())
    ms = timed(lambda: msda.sca_backward(*args5, grad_value=g5[0],
                                         grad_sampling_locations_rb=g5[1],
                                         grad_attention_weights_rb=g5[2]),
               n=max(1, iters // 4))
    r = hbm(sca_backward_algorithmic_bytes(w5, rows5, hitq5, 2), ms)
    r.update(kernel="sca_backward_kernel (+ compaction, zero fill, zero tail)",
             workload="bevformer-base SCA training step, B=2, bf16 value",
             gsamples_per_s=rows5 * w5.H * w5.L * w5.P / (ms * 1e-3) / 1e9)
    if with_cpu:
        import oracle
        nq5 = 1000
        q5 = slice(0, nq5)
        m5 = np.ascontiguousarray(w5.bev_mask[:, :, q5])
        seen5 = int(np.count_nonzero(m5.any(-1)))
        r["cpu_oracle"] = cpu_rate(
            lambda: oracle.sca_backward(w5.value, w5.spatial_shapes, w5.level_start_index,
                                        np.ascontiguousarray(w5.reference_points[:, :, q5]), m5,
                                        np.ascontiguousarray(w5.sampling_offsets[:, q5]),
                                        np.ascontiguousarray(w5.attention_logits[:, q5]),
                                        np.ascontiguousarray(w5.grad_out[:, q5])),
            seen5 * w5.H * w5.L * w5.P / 1e9, UNIT, f"the first {nq5} BEV queries")
    rows["sca_backward"] = r
    ws5 = torch.empty(int(msda.lib().sca_backward_deterministic_workspace_size(
        msda.Dims(w5.B, w5.Ncam, w5.Nq, w5.Nv, w5.H, w5.L, w5.P, w5.R))), dtype=torch.uint8,
        device="cuda")
    ms = timed(lambda: msda.sca_backward(*args5, grad_value=g5[0],
                                         grad_sampling_locations_rb=g5[1],
                                         grad_attention_weights_rb=g5[2], workspace=ws5,
                                         deterministic=True),
               n=max(1, iters // 4))
    r = hbm(sca_backward_algorithmic_bytes(w5, rows5, hitq5, 2), ms)
    r.update(kernel="sca_backward_kernel<..., deterministic> (fixed-point grad_value)",
             workload="bevformer-base SCA training step, B=2, bf16 value",
             gsamples_per_s=rows5 * w5.H * w5.L * w5.P / (ms * 1e-3) / 1e9)
    rows["sca_backward_deterministic"] = r
    # the whole backward to the SCA inputs (precise chain) in one call
    wsf = torch.empty(int(msda.lib().sca_backward_full_workspace_size(
        msda.Dims(w5.B, w5.Ncam, w5.Nq, w5.Nv, w5.H, w5.L, w5.P, w5.R))), dtype=torch.uint8,
        device="cuda")
    full_out = (g5[0], torch.empty_like(d5["off"]), torch.empty_like(d5["logits"]),
                torch.empty_like(d5["ref"]))
    ms = timed(lambda: msda.sca_backward_full(*args5, out=full_out, workspace=wsf),
               n=max(1, iters // 4))
    S5 = w5.H * w5.L * w5.P
    r = hbm(sca_backward_algorithmic_bytes(w5, rows5, hitq5, 2) - rows5 * S5 * 3 * 4
            + w5.B * w5.Nq * S5 * 3 * 4 + w5.reference_points.nbytes, ms)
    r.update(kernel="sca_backward_kernel<..., precise> + sca_offset_logit_grads_kernel "
                    "(+ compaction, zero fill)",
             workload="bevformer-base SCA training step, B=2, bf16 value",
             gsamples_per_s=rows5 * S5 / (ms * 1e-3) / 1e9)
    rows["sca_backward_full"] = r
    del wsf, full_out
    return rows


def main(argv=None):
    args = parse_args(argv)
    if args.steps < 1 or args.warmup < 3:
        raise SystemExit("need --steps >= 1 and --warmup >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
