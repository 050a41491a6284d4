#!/usr/bin/env python
"""Benchmark of the B200 W4A8 GEMM path on the decode-sweep workload.

One step = the per-call hot path for every M of the sweep N = K = 4096,
M in {1, 2, 4, 8, 16, 32, 64, 128, 256}: per-token activation quantization
of fp32 X [M, K] followed by the W4A8 GEMM with the bf16 epilogue.  The
weights are packed once, offline (LQQ weight quantization and packing are
timed separately and reported as ``offline_pack``).

* value: weight GB/s over the whole step (packed weight bytes of the nine
  GEMMs / step time), device time with CUDA events, max over ranks, one CUDA
  graph per step, 32 rotating copies of the packed weights (285 MB, more than
  twice the L2) so every GEMM streams its weights from HBM.
* roofline: the GEMM kernel, algorithmic bytes per launch / its average
  launch duration (CUDA events around graphs of back-to-back launches on the
  launching stream), against the measured HBM copy bandwidth; per-M figures
  with the bound that applies (HBM or INT8 tensor) are in ``sweep``.
* e2e: the same metric through the public calls with host buffers: each
  step uploads every M's X from one pinned host buffer, quantizes and
  multiplies (the public calls captured into CUDA graphs, as a decode loop
  replays them) and downloads every Y into one pinned host buffer.  Device buffers are double-buffered and the copies run on
  their own streams, ordered by events, so one step's upload and the
  previous step's download overlap the current step's kernels; all copies of
  every timed step are inside the timed region.
* cpu_baseline: the CPU oracle timed on a bounded sample of the same
  workload on the host cores (rank 0, one GPU only).

``--impl reference`` times the CPU oracle alone as the reference arm.
Multi-GPU (torchrun): independent replicas, one per GPU, no collective on
the data path; the step time is the max over ranks.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_block_quantized_w4a8_b200 import workloads as wl  # noqa: E402

WORKLOAD = "decode_sweep_4096"
METRIC = "W4A8 GEMM TOPS & weight GB/s vs M (1 B200), as % of INT8/HBM roofline"
UNIT = "GB/s"
N_COPIES = 32
GROUP = 64
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0  # nominal dense INT8 / bf16 tensor throughput on B200 (cross-check only)
SPEC_HBM_GBS = 8000.0  # HBM3e specification figure, for context beside the measured copy rate
# library INT8 GEMMs (cuBLASLt through torch._int_mm) whose best rate is the
# measured dense INT8 tensor peak: the square prefill shape and the two
# wide 70B-like shapes
INT8_PEAK_SHAPES = ((8192, 8192, 8192), (2048, 28672, 8192), (8192, 28672, 8192))
PDL = 1  # W4A8_FLAG_PDL: consecutive calls overlap their weight fetch with the previous kernel


# ------------------------------------------------------------------ units
def weight_bytes(N, K):
    """Packed LQQ weight bytes a GEMM must read: codes + (s_u8, a) + s_w."""
    return N * K // 2 + 2 * N * (K // GROUP) + 4 * N


def gemm_bytes(M, N, K):
    """Algorithmic HBM bytes of one GEMM: weights + Xq + s_x + Y (bf16)."""
    return weight_bytes(N, K) + M * K + 4 * M + 2 * M * N


def gemm_ops(M, N, K):
    return 2 * M * N * K


def act_bytes(M, K):
    """Activation quantization: read fp32 X, write int8 Xq and s_x."""
    return 5 * M * K + 4 * M


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS,
                    bf16_sust=1400.0, source="fallback")


def measure_int8_peak(dev, reps=10):
    """Dense INT8 tensor-core peak measured on this GPU: the best of `reps`
    runs of cuBLASLt's INT8 GEMM (torch._int_mm, INT32 output) on each shape
    of INT8_PEAK_SHAPES, timed with CUDA events; the fastest shape is the
    peak.  Returns (tops, per-shape figures)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(5)
    best, per = 0.0, []
    for M, N, K in INT8_PEAK_SHAPES:
        A = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8).to(dev)
        B = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8).to(dev)
        for _ in range(3):
            torch._int_mm(A, B.t())
        torch.cuda.synchronize(dev)
        t_best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(A, B.t())
            e1.record()
            e1.synchronize()
            t_best = min(t_best, e0.elapsed_time(e1) / 1e3)
        tops = 2.0 * M * N * K / t_best / 1e12
        per.append({"M": M, "N": N, "K": K, "us": t_best * 1e6, "tops": tops})
        best = max(best, tops)
        del A, B
    torch.cuda.empty_cache()
    return best, per


def int8_peak_tops(peaks):
    """The tensor-bound denominator: the measured INT8 peak when there is
    one, else the bf16 burst times the nominal INT8/bf16 ratio."""
    return peaks.get("int8") or peaks["bf16"] * INT8_PER_BF16


def bound_and_frac(M, N, K, seconds, peaks):
    """Roofline of one GEMM: whichever of HBM bytes and INT8 operations takes
    longer at peak, and the fraction of that time the GEMM achieved."""
    hbm_t = gemm_bytes(M, N, K) / (peaks["hbm"] * 1e9)
    tc_t = gemm_ops(M, N, K) / (int8_peak_tops(peaks) * 1e12)
    bound = "hbm" if hbm_t >= tc_t else "tensor"
    return bound, (hbm_t if bound == "hbm" else tc_t) / seconds


def bench_config():
    """The workload description shared by both arms' JSON lines."""
    layer = wl.WORKLOADS[WORKLOAD].layers[0]
    N, K = layer.N, layer.K
    return {"workload": WORKLOAD, "N": N, "K": K, "Ms": list(wl.WORKLOADS[WORKLOAD].Ms),
            "group": GROUP,
            "step": "per M: activation quantization + W4A8 GEMM (bf16 epilogue)",
            "l2": "inputs larger than L2: %d rotating packed weight copies (%.0f MB)"
                  % (N_COPIES, N_COPIES * weight_bytes(N, K) / 1e6),
            "launch": "one CUDA graph per step, programmatic dependent launch",
            "parallelism": "replicas"}


def csrc_digest():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "bit_block_quantized_w4a8_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("csrc_digest") != csrc_digest():
        return None
    return d


# ------------------------------------------------------------ distributed
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_init(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world > 1


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value, world, device=None):
    """Max of a float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(units_per_rank, world, elapsed_max_s):
    """Whole-job throughput of independent replicas: all ranks' units over
    the slowest rank's time."""
    return units_per_rank * world / elapsed_max_s


# ----------------------------------------------------------------- clocks
def gpu_local_cpus(dev):
    """The CPUs NVML reports as local to this GPU (its NUMA node), within the
    process's current affinity, or None when that cannot be read.  Pinned
    host buffers allocated while the process runs there sit in the GPU's
    local memory node, so host <-> device copies need not cross sockets."""
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(dev)
            bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            words = pynvml.nvmlDeviceGetCpuAffinity(h, ((os.cpu_count() or 1) + 63) // 64)
            cpus = {64 * i + b for i, w in enumerate(words) for b in range(64) if (w >> b) & 1}
            cpus &= os.sched_getaffinity(0)
            return cpus or None
        finally:
            pynvml.nvmlShutdown()
    except Exception:
        return None


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(p[1]), smax=float(p[2]), reasons=p[4:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        active = sorted({names[i] for r in rows for i in range(4)
                         if r["reasons"][i + 1].lower().startswith("active")})
        loaded = [r["sm"] for r in rows if r["sm"] > 0.5 * r["smax"]] or [r["sm"] for r in rows]
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": rows[0]["smax"],
                "reasons": active, "samples": len(rows)}


# ------------------------------------------------------- oracle (CPU) arm
def _oracle_inputs(Ms):
    import oracle
    layer = wl.WORKLOADS[WORKLOAD].layers[0]
    W = wl.layer_weights(WORKLOAD, layer).numpy()
    wq = oracle.quantize_weights(W, group=GROUP)
    xs = {M: wl.layer_activations(WORKLOAD, layer, M).numpy() for M in Ms}
    return wq, xs


def _rows(wq, n):
    return {k: np.ascontiguousarray(v[:n]) for k, v in wq.items()}


def _oracle_call(x, wq):
    """One oracle pass of the per-call path: activation quantization, then
    dequantization, integer GEMM and FP64 epilogue."""
    import oracle
    Xq, sx = oracle.quantize_act(x)
    oracle.w4a8_gemm(Xq, sx, wq, group=GROUP, want_acc=False)


def cpu_baseline(N, K, Ms, budget_s=12.0):
    """Oracle throughput in the bench's unit on a bounded sample: whole passes
    over the sweep's Ms (each M once per pass, increasing), repeated until
    about `budget_s` seconds of CPU time are spent (at least one pass)."""
    import oracle
    wq, xs = _oracle_inputs(Ms)
    passes, t = 0, 0.0
    while passes == 0 or t < budget_s:
        for M in Ms:
            t0 = time.perf_counter()
            _oracle_call(xs[M], wq)
            t += time.perf_counter() - t0
        passes += 1
    value = passes * len(Ms) * weight_bytes(N, K) / t / 1e9
    return {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d passes over M in %s (N=K=%d), each an oracle call: activation "
                      "quantization, dequantization, integer GEMM, FP64 epilogue"
                      % (passes, list(Ms), K),
            "seconds": t}


def run_reference(args):
    """The oracle as the reference arm, on the sample the CUDA arm's
    cpu_baseline times: each step is one pass over the sweep's nine M values
    (activation quantization, dequantization, integer GEMM, FP64 epilogue per
    M).  When warm-up and timed steps of whole passes would take longer than
    about two and a half minutes, each pass covers the first n_sub output
    channels of the layer instead (n_sub a multiple of 128)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    layer = wl.WORKLOADS[WORKLOAD].layers[0]
    N, K = layer.N, layer.K
    Ms = list(wl.WORKLOADS[WORKLOAD].Ms)
    wq, xs = _oracle_inputs(Ms)

    def one_pass(w):
        for M in Ms:
            _oracle_call(xs[M], w)
    t0 = time.perf_counter()
    one_pass(wq)
    t_full = time.perf_counter() - t0
    per_step = 150.0 / (args.steps + args.warmup)
    n_sub = N if t_full <= per_step else max(128, int(N * per_step / t_full) // 128 * 128)
    ws = wq if n_sub == N else _rows(wq, n_sub)
    for _ in range(args.warmup):
        one_pass(ws)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_pass(ws)
    t = (time.perf_counter() - t0) / args.steps
    value = len(Ms) * weight_bytes(n_sub, K) / t / 1e9
    sample = ("per step: one pass over M in %s on output channels [0, %d) of the N=K=%d layer, "
              "each an oracle call (activation quantization, dequantization, integer GEMM, "
              "FP64 epilogue)" % (Ms, n_sub, K))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": bench_config(),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- CUDA arm
def _graph(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def _time_graph(g, reps, stream):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):  # replay() launches on the current stream
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / 1e3 / reps


def run_cuda(args):
    import bit_block_quantized_w4a8_b200 as w4

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    peaks = load_peaks()
    peaks["int8"], peaks["int8_shapes"] = measure_int8_peak(dev)
    layer = wl.WORKLOADS[WORKLOAD].layers[0]
    N, K = layer.N, layer.K
    Ms = list(wl.WORKLOADS[WORKLOAD].Ms)

    # ---- offline: quantize + pack the layer once, then rotating copies
    W = wl.layer_weights(WORKLOAD, layer).to(dev)
    w4.w4a8_quantize_weights(W)  # warm-up of the packer
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    pk0 = w4.w4a8_quantize_weights(W)
    e1.record()
    e1.synchronize()
    pack_s = e0.elapsed_time(e1) / 1e3
    copies = [pk0] + [w4.PackedWeights(pk0.data.clone(), N, K, GROUP) for _ in range(N_COPIES - 1)]
    del W

    Xs = {M: wl.layer_activations(WORKLOAD, layer, M).to(dev) for M in Ms}
    Xq = {M: torch.empty(M, K, dtype=torch.int8, device=dev) for M in Ms}
    sx = {M: torch.empty(M, dtype=torch.float32, device=dev) for M in Ms}
    Ys = {M: torch.empty(M, N, dtype=torch.bfloat16, device=dev) for M in Ms}

    stream = torch.cuda.Stream(device=dev)
    # the weights were packed and copied on the default stream; the timed
    # calls run on another (non-blocking) stream
    torch.cuda.synchronize(dev)

    def step_fn(r):
        def fn():
            for j, M in enumerate(Ms):
                w4.w4a8_quantize_act(Xs[M], out=Xq[M], scale_out=sx[M], stream=stream,
                                     flags=PDL)
                w4.w4a8_gemm(Xq[M], sx[M], copies[(r * len(Ms) + j) % N_COPIES], out=Ys[M],
                             stream=stream, flags=PDL)
        return fn

    with torch.cuda.stream(stream):
        for r in range(2):  # eager warm-up: kernel attributes, tensor-map entry point
            step_fn(r)()
    stream.synchronize()
    assert w4.w4a8_get_status(stream) == 0
    n_graphs = N_COPIES
    graphs = [_graph(step_fn(r), stream) for r in range(n_graphs)]

    with torch.cuda.stream(stream):  # replay() launches on the current stream
        for s in range(args.warmup):
            graphs[s % n_graphs].replay()
    stream.synchronize()
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for s in range(args.steps):
            graphs[s % n_graphs].replay()
        t1.record(stream)
    t1.synchronize()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(world, dev)
    elapsed = t0.elapsed_time(t1) / 1e3
    elapsed_max = max_over_ranks(elapsed, world, dev)
    status = w4.w4a8_get_status(stream)
    if status != 0:
        raise RuntimeError("device status after the timed region: %s" % w4.w4a8_status_string(status))

    wbytes_step = len(Ms) * weight_bytes(N, K)
    value = replica_value(wbytes_step * args.steps, world, elapsed_max) / 1e9
    ops_step = sum(gemm_ops(M, N, K) for M in Ms)
    tops = ops_step * args.steps * world / elapsed_max / 1e12

    # ---- per-kernel durations: graphs of back-to-back launches of one kernel
    per_m = []
    reps = 10
    for M in Ms:
        def gemms(M=M, fl=PDL):
            for i in range(N_COPIES):
                w4.w4a8_gemm(Xq[M], sx[M], copies[i], out=Ys[M], stream=stream, flags=fl)

        def quants(M=M):
            for i in range(N_COPIES):
                w4.w4a8_quantize_act(Xs[M], out=Xq[M], scale_out=sx[M], stream=stream,
                                     flags=PDL)
        gg, gq = _graph(gemms, stream), _graph(quants, stream)
        g0 = _graph(lambda M=M: gemms(M, 0), stream)
        with torch.cuda.stream(stream):
            gg.replay()
            gq.replay()
            g0.replay()
        tg = _time_graph(gg, reps, stream) / N_COPIES
        tq = _time_graph(gq, reps, stream) / N_COPIES
        t_nopdl = _time_graph(g0, reps, stream) / N_COPIES
        b, o = gemm_bytes(M, N, K), gemm_ops(M, N, K)
        bound, frac = bound_and_frac(M, N, K, tg, peaks)
        T, splits, ctas = w4.w4a8_gemm_schedule(M, N, K)
        per_m.append({"M": M, "gemm_us": tg * 1e6, "gemm_us_without_pdl": t_nopdl * 1e6,
                      "act_quant_us": tq * 1e6,
                      "tops": o / tg / 1e12, "weight_gbs": weight_bytes(N, K) / tg / 1e9,
                      "total_gbs": b / tg / 1e9, "bound": bound, "frac": frac,
                      "act_quant_gbs": act_bytes(M, K) / tq / 1e9,
                      "schedule": {"tile_tokens": T, "splits": splits, "ctas": ctas}})
        del gg, gq, g0
    stream.synchronize()
    bytes_all = sum(gemm_bytes(M, N, K) for M in Ms)
    dur_all = sum(r["gemm_us"] for r in per_m) * 1e-6
    achieved = bytes_all / dur_all / 1e9
    prof = profiled_traffic()
    traffic = None
    if prof is not None:
        traffic = prof.get("sweep_mean_dram_bytes_per_launch")
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": achieved / peaks["hbm"], "traffic": traffic,
                "kernel": "w4a8_gemv_mma_kernel (M <= 16) + w4a8_gemm_kernel (M >= 32)",
                "peak_source": peaks["source"],
                "frac_of_spec": achieved / SPEC_HBM_GBS, "spec_gbs": SPEC_HBM_GBS,
                "note": "algorithmic bytes of the nine sweep launches / their summed average "
                        "launch durations"}

    # ---- e2e: public calls with host buffers, copies inside the timed region
    # One pinned host buffer holds a step's inputs (every M, stacked), one
    # its outputs.  Device inputs and outputs are double-buffered; uploads and
    # downloads run on their own streams, ordered against the compute stream
    # by events: slot b's upload waits until the compute two steps back has
    # read it, the compute waits for its upload and for the download two
    # steps back, the download waits for the compute.
    e2e_steps = max(1, min(args.steps, 200))
    offs, m_all = {}, 0
    for M in Ms:
        offs[M] = m_all
        m_all += M
    # the pinned buffers are allocated (and first written) on the GPU's local
    # CPUs, then the process's affinity is restored
    near = gpu_local_cpus(dev)
    saved_cpus = os.sched_getaffinity(0)
    if near:
        os.sched_setaffinity(0, near)
    try:
        hX = torch.empty(m_all, K, dtype=torch.float32).pin_memory()
        for M in Ms:
            hX[offs[M]:offs[M] + M].copy_(Xs[M].cpu())
        hY = [torch.empty(m_all, N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        for t in hY:
            t.zero_()
    finally:
        os.sched_setaffinity(0, saved_cpus)
    dX = [torch.empty(m_all, K, dtype=torch.float32, device=dev) for _ in range(2)]
    dY = [torch.empty(m_all, N, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # slot's upload landed
    ev_used = [torch.cuda.Event() for _ in range(2)]  # slot's kernels done
    ev_out = [torch.cuda.Event() for _ in range(2)]   # slot's download done

    # The step's calls (quantize + GEMM for every M) are captured from the
    # public API into CUDA graphs, as a decode loop replays them; four graphs
    # alternate over the two slots and rotate the weight copies, so every
    # GEMM still streams its weights from HBM.
    n_e2e = 4

    def e2e_compute(g):
        b = g % 2

        def fn():
            for j, M in enumerate(Ms):
                rows = slice(offs[M], offs[M] + M)
                xq, s_ = w4.w4a8_quantize_act(dX[b][rows], out=Xq[M], scale_out=sx[M],
                                              stream=stream, flags=PDL)
                w4.w4a8_gemm(xq, s_, copies[(g * len(Ms) + j) % N_COPIES], out=dY[b][rows],
                             stream=stream, flags=PDL)
        return fn

    e2e_graphs = [_graph(e2e_compute(g), stream) for g in range(n_e2e)]

    def e2e_step(r):
        b = r % 2
        s_in.wait_event(ev_used[b])
        with torch.cuda.stream(s_in):
            dX[b].copy_(hX, non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])
        with torch.cuda.stream(stream):
            e2e_graphs[r % n_e2e].replay()
        ev_used[b].record(stream)
        s_out.wait_event(ev_used[b])
        with torch.cuda.stream(s_out):
            hY[b].copy_(dY[b], non_blocking=True)
        ev_out[b].record(s_out)

    for r in range(3):
        e2e_step(r)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    s_in.wait_event(a0)
    for r in range(e2e_steps):
        e2e_step(r)
    for b in range(2):  # the last two downloads are part of the run
        stream.wait_event(ev_out[b])
    a1.record(stream)
    a1.synchronize()
    torch.cuda.synchronize(dev)
    # the weight copies are identical, so the downloaded outputs of the last
    # step equal the graph run's: a check on the pipeline's ordering
    last = hY[(e2e_steps - 1) % 2]
    for M in Ms:
        if not torch.equal(last[offs[M]:offs[M] + M].view(torch.int16),
                           Ys[M].cpu().view(torch.int16)):
            raise RuntimeError("e2e outputs differ from the timed run's at M=%d" % M)
    e2e_el = max_over_ranks(a0.elapsed_time(a1) / 1e3, world, dev)
    e2e_value = replica_value(wbytes_step * e2e_steps, world, e2e_el) / 1e9
    h2d = sum(M * K * 4 for M in Ms)
    d2h = sum(M * N * 2 for M in Ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(N, K, Ms, budget_s=args.cpu_budget)

    # ---- every workload's cases (kernel timings, clocks sampled throughout);
    # one GPU only, outside the timed region
    all_cfg = None
    if world == 1 and not args.no_all_configs:
        del graphs[:], e2e_graphs[:]
        copies.clear()
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        ck = ClockSampler(local)
        ck.start()
        cases = time_all_cases(w4, dev, stream, peaks)
        all_cfg = {"clocks": ck.stop(), "targets": target_summary(cases),
                   "timing": "each case a CUDA graph of back-to-back launches with programmatic "
                             "dependent launch over rotating weight copies larger than twice the "
                             "L2; CUDA events on the launching stream",
                   "cases": [{k: c[k] for k in ("workload", "layer", "M", "N", "K", "gemm_us",
                                                "tops", "weight_gbs", "bound", "frac",
                                                "act_quant_us", "status", "schedule")}
                             for c in cases]}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed_max / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": bench_config(),
        "tops": tops,
        "gpu_launches": 2 * len(Ms) * args.steps,
        "roofline": roofline,
        "sweep": per_m,
        "offline_pack": {"seconds": pack_s, "fp32_weight_gbs": 4 * N * K / pack_s / 1e9},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipeline": "one upload and one download per step on their own streams, "
                            "double-buffered against the compute stream; the step's public "
                            "calls replayed from CUDA graphs",
                "host_buffers": ("pinned, allocated on the GPU's local CPUs (%d)" % len(near))
                                if near else "pinned, default placement"},
        "clocks": clk,
        "cpu_baseline": cpu,
        "peaks": {"hbm_gbs": peaks["hbm"], "hbm_source": peaks["source"],
                  "int8_tops": peaks["int8"],
                  "int8_source": "measured: best cuBLASLt INT8 GEMM (torch._int_mm) of %s"
                                 % ["%dx%dx%d" % (d["M"], d["N"], d["K"])
                                    for d in peaks["int8_shapes"]],
                  "int8_shapes": peaks["int8_shapes"],
                  "int8_nominal_from_bf16": peaks["bf16"] * INT8_PER_BF16},
        "all_configs": all_cfg,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    graphs.clear()
    e2e_graphs.clear()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_profile_case(args):
    """Small fixed case for profilers: pack one layer (default: the N=K=4096
    decode layer; --profile-layer WORKLOAD:LAYER for another) and run one
    GEMM per requested M (no graphs, no timing)."""
    import bit_block_quantized_w4a8_b200 as w4
    torch.cuda.set_device(0)
    name, lname = (args.profile_layer or WORKLOAD + ":square").split(":")
    layer = [L for L in wl.WORKLOADS[name].layers if L.name == lname][0]
    pk = w4.w4a8_quantize_weights(wl.layer_weights(name, layer).cuda())
    for M in [int(x) for x in args.profile.split(",")]:
        Xq, sx = w4.w4a8_quantize_act(wl.layer_activations(name, layer, M).cuda())
        w4.w4a8_gemm(Xq, sx, pk)
    torch.cuda.synchronize()
    status = w4.w4a8_get_status()
    print("profile case done, status %s" % w4.w4a8_status_string(status))
    return 0 if status == 0 else 1


def time_all_cases(w4, dev, stream, peaks, verbose=True):
    """Kernel timings on every synthetic workload (all layers and M values):
    per case the GEMM and the activation quantizer are each timed as graphs
    of back-to-back launches (programmatic dependent launch), with enough
    rotating weight copies that the working set exceeds twice the L2.
    Returns one dict per case."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    cases = []
    for name in wl.WORKLOADS:
        layers_done = {}
        for M, layer in wl.cases(name):
            N, K = layer.N, layer.K
            if layer.name not in layers_done:
                layers_done.clear()
                torch.cuda.empty_cache()
                W = wl.layer_weights(name, layer).to(dev)
                pk = w4.w4a8_quantize_weights(W)
                del W
                ncopy = max(1, min(32, -(-2 * l2 // pk.data.numel())))
                copies = [pk] + [w4.PackedWeights(pk.data.clone(), N, K, GROUP)
                                 for _ in range(ncopy - 1)]
                torch.cuda.synchronize(dev)  # packed on the default stream; timed calls on another
                layers_done[layer.name] = copies
            copies = layers_done[layer.name]
            X = wl.layer_activations(name, layer, M).to(dev)
            Xq = torch.empty(M, K, dtype=torch.int8, device=dev)
            sx = torch.empty(M, dtype=torch.float32, device=dev)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            reps_in = max(len(copies), 4)
            with torch.cuda.stream(stream):
                w4.w4a8_quantize_act(X, out=Xq, scale_out=sx, stream=stream)
                w4.w4a8_gemm(Xq, sx, copies[0], out=Y, stream=stream)
            stream.synchronize()

            def gemms():
                for i in range(reps_in):
                    w4.w4a8_gemm(Xq, sx, copies[i % len(copies)], out=Y, stream=stream,
                                 flags=PDL)

            def quants():
                for i in range(reps_in):
                    w4.w4a8_quantize_act(X, out=Xq, scale_out=sx, stream=stream, flags=PDL)
            gg, gq = _graph(gemms, stream), _graph(quants, stream)
            with torch.cuda.stream(stream):
                gg.replay()
                gq.replay()
            reps = max(3, min(50, int(2e-3 / max(1e-6, _time_graph(gg, 1, stream)))))
            tg = _time_graph(gg, reps, stream) / reps_in
            tq = _time_graph(gq, reps, stream) / reps_in
            status = w4.w4a8_get_status(stream)
            b, o = gemm_bytes(M, N, K), gemm_ops(M, N, K)
            bound, frac = bound_and_frac(M, N, K, tg, peaks)
            T, splits, ctas = w4.w4a8_gemm_schedule(M, N, K)
            case = {"workload": name, "layer": layer.name, "M": M, "N": N, "K": K,
                    "gemm_us": tg * 1e6, "tops": o / tg / 1e12,
                    "weight_gbs": weight_bytes(N, K) / tg / 1e9, "total_gbs": b / tg / 1e9,
                    "bound": bound, "frac": frac,
                    "act_quant_us": tq * 1e6, "act_quant_gbs": act_bytes(M, K) / tq / 1e9,
                    "weight_copies": len(copies), "status": status,
                    "schedule": {"tile_tokens": T, "splits": splits, "ctas": ctas}}
            cases.append(case)
            if verbose:
                print("%-18s %-9s M=%-6d %9.2f us %8.1f TOPS %7.0f wGB/s %-6s %.3f  (%s)" % (
                    name, layer.name, M, case["gemm_us"], case["tops"], case["weight_gbs"],
                    bound, case["frac"], case["schedule"]), file=sys.stderr, flush=True)
            del gg, gq, X, Xq, sx, Y
        layers_done.clear()
    torch.cuda.empty_cache()
    return cases


def target_summary(cases):
    """The two targets over the timed cases: HBM fraction at M <= 16 and INT8
    tensor fraction at M >= 4096 (lowest and highest of each).  The HBM target
    is about LLM-layer shapes, so the tiny correctness case (N=256, K=512: 70 KB
    of weights, a launch's latency whatever the kernel) is left out of it and
    named in the summary."""
    small = [c["frac"] for c in cases
             if c["M"] <= 16 and c["bound"] == "hbm" and c["workload"] != "tiny"]
    large = [c["frac"] for c in cases if c["M"] >= 4096 and c["bound"] == "tensor"]
    out = {}
    if small:
        out["hbm_frac_at_M_le_16"] = {"min": min(small), "max": max(small), "cases": len(small),
                                      "target": 0.70, "excluded": "tiny (correctness case)"}
    if large:
        out["int8_frac_at_M_ge_4096"] = {"min": min(large), "max": max(large),
                                         "cases": len(large), "target": 0.60}
    return out


def run_all_configs(args):
    """--all-configs PATH: every workload case timed (``time_all_cases``),
    the INT8 peak measured first and the clocks sampled throughout; one JSON
    document to PATH."""
    import bit_block_quantized_w4a8_b200 as w4
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    peaks["int8"], peaks["int8_shapes"] = measure_int8_peak(dev)
    stream = torch.cuda.Stream(device=dev)
    clocks = ClockSampler(0)
    clocks.start()
    cases = time_all_cases(w4, dev, stream, peaks)
    out = {"peaks": peaks, "clocks": clocks.stop(), "cases": cases,
           "targets": target_summary(cases)}
    with open(args.all_configs, "w") as f:
        json.dump(out, f, indent=1)
    return 0


def run_compare(args):
    """The pages' comparison points on one harness (each timed as a graph of
    back-to-back calls over rotating weight copies larger than twice the L2):
    this library's W4A8 GEMM with group 64 and group 128, its W8A8 kernel
    (INT8 weights, same rings and epilogue, no dequantization), and two
    library references -- cuBLASLt INT8 (torch._int_mm: INT32 output, no
    epilogue; M padded to 32 rows where it needs more than 16) and cuBLAS
    bf16 (torch.mm on unquantized weights).  Writes JSON to ``args.compare``."""
    import bit_block_quantized_w4a8_b200 as w4
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    peaks["int8"], peaks["int8_shapes"] = measure_int8_peak(dev)
    clocks = ClockSampler(0)
    clocks.start()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.Stream(device=dev)
    shapes = [("decode_sweep_4096", "square", [1, 4, 16, 64, 128, 256]),
              ("llama7b_like", "qkv", [1, 16, 128, 1024]),
              ("llama70b_like", "up", [1, 32, 512, 2048]),
              ("llama70b_like", "down", [1, 32, 512, 2048])]
    out = {"peaks": peaks, "cases": []}

    def copies_of(t, nbytes):
        n = max(1, min(32, -(-2 * l2 // nbytes)))
        cs = [t] + [t.clone() for _ in range(n - 1)]
        torch.cuda.synchronize(dev)  # clones on the default stream; timed calls on another
        return cs

    def timed(fn_i, n_in):
        def body():
            for i in range(n_in):
                fn_i(i)
        with torch.cuda.stream(stream):
            fn_i(0)
        stream.synchronize()
        g = _graph(body, stream)
        with torch.cuda.stream(stream):
            g.replay()
        reps = max(3, min(50, int(2e-3 / max(1e-6, _time_graph(g, 1, stream)))))
        t = _time_graph(g, reps, stream) / n_in
        del g
        return t

    for name, lname, Ms in shapes:
        layer = [L for L in wl.WORKLOADS[name].layers if L.name == lname][0]
        N, K = layer.N, layer.K
        torch.cuda.empty_cache()
        W = wl.layer_weights(name, layer).to(dev)
        pk64 = w4.w4a8_quantize_weights(W, group=64)
        pk128 = w4.w4a8_quantize_weights(W, group=128)
        Wq, sw = w4.w8a8_quantize_weights(W)
        Wbf = W.to(torch.bfloat16)
        del W
        c64 = copies_of(pk64.data, pk64.data.numel())
        c128 = copies_of(pk128.data, pk128.data.numel())
        c8 = copies_of(Wq, Wq.numel())
        cbf = copies_of(Wbf, 2 * Wbf.numel())
        p64 = [w4.PackedWeights(d, N, K, 64) for d in c64]
        p128 = [w4.PackedWeights(d, N, K, 128) for d in c128]
        for M in Ms:
            X = wl.layer_activations(name, layer, M).to(dev)
            Xq, sx = w4.w4a8_quantize_act(X)
            Xbf = X.to(torch.bfloat16)
            Mp = M if M > 16 else 32
            Xq_p = torch.zeros(Mp, K, dtype=torch.int8, device=dev)
            Xq_p[:M] = Xq
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            n_in = 8
            t = {}
            t["w4a8_g64"] = timed(lambda i: w4.w4a8_gemm(Xq, sx, p64[i % len(p64)], out=Y,
                                                         stream=stream, flags=PDL), n_in)
            t["w4a8_g128"] = timed(lambda i: w4.w4a8_gemm(Xq, sx, p128[i % len(p128)], out=Y,
                                                          stream=stream, flags=PDL), n_in)
            t["w8a8"] = timed(lambda i: w4.w8a8_gemm(Xq, sx, c8[i % len(c8)], sw, out=Y,
                                                     stream=stream, flags=PDL), n_in)
            t["cublaslt_int8_i32"] = timed(lambda i: torch._int_mm(Xq_p, c8[i % len(c8)].t()),
                                           n_in)
            t["cublas_bf16"] = timed(lambda i: torch.mm(Xbf, cbf[i % len(cbf)].t()), n_in)
            status = w4.w4a8_get_status(stream)
            o = gemm_ops(M, N, K)
            case = {"workload": name, "layer": lname, "M": M, "N": N, "K": K, "status": status,
                    "us": {k: v * 1e6 for k, v in t.items()},
                    "tops": {k: o / v / 1e12 for k, v in t.items()},
                    "w4a8_speedup": {k: v / t["w4a8_g64"] for k, v in t.items()},
                    "m_padded_for_int_mm": Mp}
            out["cases"].append(case)
            print("%-18s %-6s M=%-5d " % (name, lname, M) + "  ".join(
                "%s %.2fus" % (k, v * 1e6) for k, v in t.items()), flush=True)
        del c64, c128, c8, cbf, p64, p128, pk64, pk128, Wq, sw, Wbf
    out["clocks"] = clocks.stop()
    with open(args.compare, "w") as f:
        json.dump(out, f, indent=1)
    return 0


def run_moe(args):
    """The grouped (mixture-of-experts) GEMM on the Mixtral-like expert layers
    (8 experts, top-2): one grouped launch per layer call, against one dense
    launch per expert that has rows.  Both timed as graphs of back-to-back
    calls (programmatic dependent launch) over rotating copies of the expert
    weights, with at least twice the L2 of active expert bytes.  Writes JSON
    to ``args.moe``."""
    import bit_block_quantized_w4a8_b200 as w4
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    peaks["int8"], peaks["int8_shapes"] = measure_int8_peak(dev)
    clocks = ClockSampler(0)
    clocks.start()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.Stream(device=dev)
    name = "mixtral_like"
    w = wl.MOE_WORKLOADS[name]
    out = {"peaks": peaks, "workload": name, "cases": []}
    for layer in w.layers:
        N, K = layer.N, layer.K
        b = w4.w4a8_packed_weight_bytes(N, K)
        torch.cuda.empty_cache()
        data = torch.empty(w.experts * b, dtype=torch.uint8, device=dev)
        for e in range(w.experts):
            w4.w4a8_quantize_weights(wl.moe_expert_weights(name, layer, e).to(dev),
                                     out=data[e * b:(e + 1) * b])
        for tokens in w.tokens:
            offsets, tok = wl.moe_routing(name, tokens)
            o = offsets.tolist()
            active = [e for e in range(w.experts) if o[e + 1] > o[e]]
            act_bytes = len(active) * weight_bytes(N, K)
            ncopy = max(1, min(4, -(-2 * l2 // act_bytes)))
            copies = [data] + [data.clone() for _ in range(ncopy - 1)]
            torch.cuda.synchronize(dev)  # packed on the default stream; timed calls on another
            gws = [w4.GroupedPackedWeights(d, w.experts, N, K, GROUP) for d in copies]
            X = wl.moe_activations(name, layer, tokens)[tok].contiguous().to(dev)
            M = X.shape[0]
            Xq, sx = w4.w4a8_quantize_act(X)
            off = offsets.to(dev)
            mr = max(o[e + 1] - o[e] for e in range(w.experts))
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            n_in = 8

            def grouped():
                for i in range(n_in):
                    w4.w4a8_grouped_gemm(Xq, sx, gws[i % ncopy], off, max_rows=mr, out=Y,
                                         stream=stream, flags=PDL)

            views = [(o[e], o[e + 1], [g.expert(e) for g in gws]) for e in active]

            def per_expert():
                for i in range(n_in):
                    for r0, r1, ex in views:
                        w4.w4a8_gemm(Xq[r0:r1], sx[r0:r1], ex[i % ncopy], out=Y[r0:r1],
                                     stream=stream, flags=PDL)
            t = {}
            for key, fn in (("grouped", grouped), ("per_expert_dense", per_expert)):
                with torch.cuda.stream(stream):
                    fn()
                stream.synchronize()
                g = _graph(fn, stream)
                with torch.cuda.stream(stream):
                    g.replay()
                reps = max(3, min(50, int(2e-3 / max(1e-6, _time_graph(g, 1, stream)))))
                t[key] = _time_graph(g, reps, stream) / n_in
                del g
            status = w4.w4a8_get_status(stream)
            ops = 2.0 * M * N * K
            tot_bytes = act_bytes + M * K + 4 * M + 2 * M * N
            hbm_t, tc_t = tot_bytes / (peaks["hbm"] * 1e9), ops / (int8_peak_tops(peaks) * 1e12)
            bound = "hbm" if hbm_t >= tc_t else "tensor"
            tg = t["grouped"]
            T, splits, ctas = w4.w4a8_grouped_gemm_schedule(w.experts, M, mr, N, K)
            case = {"layer": layer.name, "tokens": tokens, "rows": M, "N": N, "K": K,
                    "active_experts": len(active), "max_rows": mr, "status": status,
                    "grouped_us": tg * 1e6, "per_expert_dense_us": t["per_expert_dense"] * 1e6,
                    "speedup_vs_per_expert": t["per_expert_dense"] / tg,
                    "active_weight_gbs": act_bytes / tg / 1e9, "tops": ops / tg / 1e12,
                    "bound": bound, "frac": (hbm_t if bound == "hbm" else tc_t) / tg,
                    "schedule": {"tile_tokens": T, "splits": splits, "ctas": ctas},
                    "weight_copies": ncopy}
            out["cases"].append(case)
            print("%-8s tokens=%-4d rows=%-5d experts=%d grouped %8.2f us  per-expert %8.2f us  "
                  "x%.2f  %7.0f wGB/s %7.1f TOPS %-6s %.3f %s" % (
                      layer.name, tokens, M, len(active), tg * 1e6,
                      t["per_expert_dense"] * 1e6, case["speedup_vs_per_expert"],
                      case["active_weight_gbs"], case["tops"], bound, case["frac"],
                      case["schedule"]), flush=True)
            del copies, gws
        del data
    out["clocks"] = clocks.stop()
    with open(args.moe, "w") as f:
        json.dump(out, f, indent=1)
    return 0


def run_ablation(args):
    """The ablation study: each kernel variant of ``w4a8_gemm_variant``
    (one design decision changed against a fixed baseline) timed on decode,
    mid-size and prefill shapes, as graphs of back-to-back calls
    (programmatic dependent launch) over rotating weight copies larger than
    twice the L2.  Writes JSON to ``args.ablation``."""
    import bit_block_quantized_w4a8_b200 as w4
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    peaks["int8"], peaks["int8_shapes"] = measure_int8_peak(dev)
    clocks = ClockSampler(0)
    clocks.start()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.Stream(device=dev)
    shapes = [("decode_sweep_4096", "square", [1, 16, 256]),
              ("llama70b_like", "up", [1]),
              ("llama70b_like", "down", [512]),
              ("prefill", "square8k", [8192])]
    variants = ["default", "baseline", "naive_dequant", "serial", "one_group",
                "group_issues_mma", "cta_pair", "tensor_core", "warp_mma", "dp4a", "persistent"]
    out = {"peaks": peaks, "variants": variants, "cases": []}
    for name, lname, Ms in shapes:
        layer = [L for L in wl.WORKLOADS[name].layers if L.name == lname][0]
        N, K = layer.N, layer.K
        torch.cuda.empty_cache()
        pk = w4.w4a8_quantize_weights(wl.layer_weights(name, layer).to(dev))
        ncopy = max(1, min(32, -(-2 * l2 // pk.data.numel())))
        copies = [pk] + [w4.PackedWeights(pk.data.clone(), N, K, GROUP) for _ in range(ncopy - 1)]
        torch.cuda.synchronize(dev)  # packed on the default stream; timed calls on another
        for M in Ms:
            X = wl.layer_activations(name, layer, M).to(dev)
            Xq, sx = w4.w4a8_quantize_act(X)
            del X
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            n_in = 8 if M < 4096 else 2
            t = {}
            for v in variants:
                if v in ("cta_pair", "persistent") and (M < 256 or (-(-N // 128)) % 2):
                    continue  # the pair forms need full 256-token tiles, paired channel blocks
                if (v == "warp_mma" and M > 16) or (v == "dp4a" and M > 8):
                    continue  # the decode form's token limits
                if v == "tensor_core" and M > 16:
                    continue  # the default is the tensor-core kernel already
                def body(v=v):
                    for i in range(n_in):
                        w4.w4a8_gemm_variant(v, Xq, sx, copies[i % ncopy], out=Y, stream=stream,
                                             flags=PDL)
                with torch.cuda.stream(stream):
                    body()
                stream.synchronize()
                g = _graph(body, stream)
                with torch.cuda.stream(stream):
                    g.replay()
                reps = max(3, min(50, int(2e-3 / max(1e-6, _time_graph(g, 1, stream)))))
                t[v] = _time_graph(g, reps, stream) / n_in
                del g
            status = w4.w4a8_get_status(stream)
            base = t["baseline"]
            case = {"workload": name, "layer": lname, "M": M, "N": N, "K": K, "status": status,
                    "us": {k: x * 1e6 for k, x in t.items()},
                    "vs_baseline": {k: x / base for k, x in t.items()},
                    "tops": {k: gemm_ops(M, N, K) / x / 1e12 for k, x in t.items()}}
            out["cases"].append(case)
            print("%-18s %-9s M=%-5d " % (name, lname, M) + "  ".join(
                "%s %.2fus" % (k, x * 1e6) for k, x in t.items()), flush=True)
        del copies, pk
    out["clocks"] = clocks.stop()
    with open(args.ablation, "w") as f:
        json.dump(out, f, indent=1)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-all-configs", action="store_true",
                    help="skip the per-case timings of every workload after the timed run")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of CPU work for the oracle baseline sample")
    ap.add_argument("--profile", default=None,
                    help="comma-separated Ms: run one GEMM each on N=K=4096 for a profiler")
    ap.add_argument("--profile-layer", default=None, metavar="WORKLOAD:LAYER",
                    help="layer for --profile (default decode_sweep_4096:square)")
    ap.add_argument("--all-configs", default=None, metavar="PATH",
                    help="time every workload case and write a JSON report to PATH")
    ap.add_argument("--compare", default=None, metavar="PATH",
                    help="time W4A8 (group 64/128), W8A8 and library GEMMs side by side; "
                         "write a JSON report to PATH")
    ap.add_argument("--moe", default=None, metavar="PATH",
                    help="time the grouped (mixture-of-experts) GEMM on the Mixtral-like "
                         "layers; write a JSON report to PATH")
    ap.add_argument("--ablation", default=None, metavar="PATH",
                    help="time the kernel variants of the ablation study; write JSON to PATH")
    args = ap.parse_args(argv)
    if args.ablation:
        return run_ablation(args)
    if args.moe:
        return run_moe(args)
    if args.compare:
        return run_compare(args)
    if args.all_configs:
        return run_all_configs(args)
    if args.profile:
        return run_profile_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
