"""Benchmark of the NVFP4 W4A4 routed-MoE feed-forward layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode] [--impl ours|reference]

One step = one full pass of the layer (route, permute, quantise x, gate/up + SwiGLU +
requantise, down, combine) over one batch of synthetic tokens, inputs resident in HBM,
timed as a replay of the forward captured once into a CUDA graph (the kernels and buffers of
an eager call, without the host's per-launch gaps).  L2 is flushed before every timed step (a 256 MiB write, then a 256 MiB read so the step
starts from a clean, cold L2), outside the timed events.
Prints one JSON line on rank 0.  With N > 1 (torchrun) every rank runs an independent
replica on its own GPU (the layer has no cross-GPU exchange on one device's batch), the
timed region is bracketed by barriers and the reported time is the max over ranks.

--impl reference times the CPU oracle (the plain C++ implementation the tests check
against) on the machine's host cores on the same workload: a deliberately slow baseline.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_mixture_experts_w4a4_b200 import _lib as C  # noqa: E402
from nvfp4_mixture_experts_w4a4_b200 import ops, workloads as W  # noqa: E402

METRIC = "NVFP4 MoE-layer tokens/s; % of HBM BW (decode) / % FP4 TC peak (prefill)"
FP4_BYTES_PER_ELT = 0.5625  # 4-bit code + one E4M3 scale per 16 elements
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Leaves L2 cold before a timed step: writes a 256 MiB buffer (evicting everything),
    then reads another 256 MiB buffer so the write-backs of those dirty lines happen here,
    outside the timed events, and the step starts from a clean, cold L2 (as after a previous
    layer's weight reads) instead of paying for the flush's own write-backs."""

    def __init__(self, dev):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.sink = torch.empty((), dtype=torch.int32, device=dev)

    def zero_(self):
        self.w.zero_()
        torch.amax(self.r, dim=0, out=self.sink)
        return self


def peaks(dev=None):
    """Roofline denominators: HBM copy and bf16 GEMM from MEASURED_PEAKS.json (or the pool's
    fallback figures), and the dense FP4 tensor peak measured on this device by the library's
    tcgen05 kind::mxf4nvf4 MMA loop (operands resident in shared memory) when a device is
    given, else the bf16 burst figure times the nominal FP4/BF16 ratio (9 / 2.25)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        pk = {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
              "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    else:
        pk = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    pk["fp4_tflops"] = pk["bf16_tflops"] * 4.0
    pk["fp4_source"] = "bf16 burst x 4"
    if dev is not None:
        pk["fp4_tflops"] = ops.mma_peak_tflops()
        pk["fp4_source"] = ("measured: tcgen05 mxf4nvf4 MMA loop, M128 N256 K64, one CTA per SM, operands "
                            "resident in shared memory")
    return pk


# tokens of the workload the oracle runs per CPU-baseline pass / reference step
ORACLE_SAMPLE = {"tiny": 8, "decode": 16, "prefill_chunk": 16, "long_prefill": 4, "dense": 2, "dense_t1": 1}


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons of this rank's GPU, sampled through NVML
    every millisecond while the timed region runs (nvidia-smi's fastest period is too coarse
    for a region of a few milliseconds)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, cuda_index: int, period_s: float = 0.001):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml as N
            N.nvmlInit()
            props = torch.cuda.get_device_properties(self.cuda_index)
            busid = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self.h = N.nvmlDeviceGetHandleByPciBusId_v2(busid)
            except Exception:
                self.h = N.nvmlDeviceGetHandleByIndex(self.cuda_index)
            self.N = N
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self.stop = threading.Event()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        return self

    def _reasons(self):
        N = self.N
        try:
            return N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return N.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        N = self.N
        while not self.stop.is_set():
            try:
                self.samples.append((N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM), self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        if self.ok:
            self.stop.set()
            self.t.join(timeout=2)

    def summary(self):
        sm = [c for c, _ in self.samples]
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvml" if self.ok else "unavailable"}


def setup_layer(wl: W.Workload, dev, seed: int = 0, path: int = C.PATH_AUTO, launch: int = C.LAUNCH_AUTO):
    """Draws the workload on the device, quantises the weights with the library, and
    calibrates the per-expert requantisation scales with one forward (h_amax / 2688)."""
    act = W.make_activations(wl, seed, dev)
    wts = W.make_weights(wl, seed, dev)
    experts = ops.NVFP4Experts.from_float(wts["w_gate"], wts["w_up"], wts["w_down"])
    del wts
    ones = torch.ones(wl.E, dtype=torch.float32, device=dev)
    layer = ops.MoeFFN(experts, wl.k, ones, path=path, launch=launch)
    h_amax = torch.empty(wl.E, dtype=torch.float32, device=dev)
    layer(act["x"], act["logits"], h_amax=h_amax)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    s_h = torch.where(h_amax > 0, h_amax / 2688.0, ones)
    layer = ops.MoeFFN(experts, wl.k, s_h, path=path, launch=launch)
    return act, experts, layer


def algorithmic(wl: W.Workload, n_active: int, gemm_path: bool, a16: bool = False, shared_I: int = 0):
    """Algorithmic (compulsory) bytes and FLOPs of one layer pass and of its gate/up stage:
    each touched expert's weights once, the quantised activations once (per permuted row on
    the tensor-core path, which gathers x into expert order), h written and read once.
    Weight-only (a16): x and h in bf16.  A shared expert adds its bf16 weights and its FLOPs to
    the layer (not to the gate/up stage)."""
    e = FP4_BYTES_PER_ELT
    P = wl.T * wl.k
    w13 = n_active * 2 * wl.I * wl.H * e
    w2 = n_active * wl.H * wl.I * e
    x_q = (P if gemm_path else wl.T) * wl.H * (2 if a16 else e)
    h_q = P * wl.I * (2 if a16 else e)
    gate_up_bytes = w13 + x_q + h_q
    layer_bytes = w13 + w2 + wl.T * wl.H * 2 * 2 + x_q + 2 * h_q + wl.T * wl.E * 4 + 3 * wl.H * shared_I * 2
    flops = 2.0 * P * 3 * wl.H * wl.I + 2.0 * wl.T * 3 * wl.H * shared_I
    # both GEMMs in one launch (small batches): weights, x and h codes, fp32 slot rows
    gemms_bytes = w13 + w2 + x_q + 2 * h_q + P * wl.H * 4
    return {"gate_up_bytes": gate_up_bytes, "layer_bytes": layer_bytes, "flops": flops,
            "gate_up_flops": 2.0 * P * 2 * wl.H * wl.I, "gemms_bytes": gemms_bytes}


# nominal B200 figures, for the fractions quoted beside the measured ones: HBM3e at 8 TB/s and
# the published dense FP4 tensor peak (9 PFLOP/s; the doubled figure assumes 2:4 sparsity)
NOMINAL_HBM_GBS = 8000.0
NOMINAL_FP4_TFLOPS = 9000.0


def roofline(bytes_, flops, ms, pk):
    """Binding roofline of a kernel that moves `bytes_` and does `flops` in `ms`: the fraction
    of the measured peak, and beside it the fraction of the nominal one."""
    t_hbm = bytes_ / (pk["hbm_gbs"] * 1e9)
    t_tc = flops / (pk["fp4_tflops"] * 1e12)
    if t_hbm >= t_tc:
        ach = bytes_ / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
                "nominal": {"peak": NOMINAL_HBM_GBS, "frac": ach / NOMINAL_HBM_GBS}}
    ach = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": pk["fp4_tflops"], "unit": "TFLOP/s",
            "frac": ach / pk["fp4_tflops"], "nominal": {"peak": NOMINAL_FP4_TFLOPS, "frac": ach / NOMINAL_FP4_TFLOPS}}


def capture_layer(layer, act, out, stage_events=None):
    """The layer's forward captured once into a CUDA graph (with its stage marks as timing
    nodes when stage_events is given); replays launch the same kernels on the same buffers."""
    if stage_events is not None:
        for e in stage_events:
            e.record()  # materialise the events outside the capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.stream(s):
        layer(act["x"], act["logits"], out=out)
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            layer(act["x"], act["logits"], out=out, stage_events=stage_events)
    torch.cuda.current_stream().wait_stream(s)
    g.instantiate()
    torch.cuda.synchronize()
    return g


def kernel_nodes(g) -> int | None:
    """Number of kernel launches in a captured graph (None when cuda-python cannot tell)."""
    try:
        from cuda.bindings import runtime as rt
        graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
        err, nodes, n = rt.cudaGraphGetNodes(graph, numNodes=0)
        err, nodes, n = rt.cudaGraphGetNodes(graph, numNodes=n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes[:n]]
        return sum(1 for t in kinds if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:  # noqa: BLE001 - an introspection failure only loses the count
        return None


def measured_traffic(workload: str, source: str = "ffn_grouped.cu"):
    """DRAM bytes per launch of the dominant kernel from the committed ncu capture of this
    workload, or None when there is none or the kernel's source file changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f).get(workload)
        src = os.path.join(ROOT, "nvfp4_mixture_experts_w4a4_b200", "csrc", source)
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha256") != digest or rec.get("source", "ffn_grouped.cu") != source:
        return None
    return rec["dram_read_bytes"] + rec["dram_write_bytes"]


def max_over_ranks(x: float) -> float:
    """The max of a per-rank time over all ranks (identity without a process group).  Uses a
    CPU tensor under gloo and a device tensor under nccl."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    dev = "cpu" if torch.distributed.get_backend() == "gloo" else torch.device("cuda", torch.cuda.current_device())
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(total_ms_max: float, steps: int, world: int, tokens_per_rank: int):
    """(ms per step, whole-job tokens/s): every rank processes its own batch of tokens_per_rank
    tokens per step, and the job's step time is the slowest rank's."""
    ms_per_step = total_ms_max / steps
    return ms_per_step, world * tokens_per_rank / (ms_per_step * 1e-3)


def time_steps(layer, act, steps: int, warmup: int, flush: L2Flush, dist_on: bool):
    """Device time of K layer passes, each a replay of the captured forward between CUDA
    events on the replay stream, L2 flushed before each; then K more replays of a capture that
    carries the stage marks, for the per-stage split (its marks cost a little time each)."""
    out = torch.empty(act["x"].shape[0], layer.w.H, dtype=torch.bfloat16, device=act["x"].device)
    g = capture_layer(layer, act, out)
    launches = kernel_nodes(g)
    for _ in range(warmup):
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush.zero_()
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]

    marks = [torch.cuda.Event(enable_timing=True) for _ in range(C.STAGES)]
    gs = capture_layer(layer, act, out, stage_events=marks)
    per_stage = {name: [] for name in C.STAGE_NAMES}
    for i in range(warmup + steps):
        flush.zero_()
        gs.replay()
        torch.cuda.synchronize()
        if i >= warmup:
            for j, name in enumerate(C.STAGE_NAMES):
                per_stage[name].append(marks[j].elapsed_time(marks[j + 1]))
    stage_ms = {name: statistics.mean(v) for name, v in per_stage.items()}
    del g, gs
    return step_ms, stage_ms, launches


def time_e2e(layer, act, steps: int, warmup: int, flush: torch.Tensor):
    """The same pass through the public API with host buffers: the graphed layer
    (ops.GraphedMoeFFN with host_io) copies x and logits from its pinned host inputs to the
    device, runs, and copies the output back to its pinned host output, all in one replay
    inside the events."""
    graphed = ops.GraphedMoeFFN(layer, act["x"].shape[0], host_io=True)
    graphed.x_host.copy_(act["x"].cpu())
    graphed.logits_host.copy_(act["logits"].cpu())
    ms = []
    for i in range(warmup + steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graphed()
        b.record()
        b.synchronize()
        if i >= warmup:
            ms.append(a.elapsed_time(b))
    h2d = sum(t.numel() * t.element_size() for t in (graphed.x_host, graphed.logits_host))
    d2h = graphed.out_host.numel() * graphed.out_host.element_size()
    return statistics.mean(ms), h2d, d2h


# ----------------------------------------------------------- oracle (CPU) ----
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_inputs(wl: W.Workload, n: int, seed: int = 0):
    """Inputs of the oracle's timed leg, drawn on the host alone: the workload's activations
    (same recipe as the device's, from the CPU generator), the first n tokens, and the oracle's
    own quantisation of the fp32 weights of every expert those tokens select, each expert
    drawn by workloads.make_expert_weights.  Nothing here touches the GPU or the library."""
    import oracle as O
    act = W.make_activations(wl, seed, "cpu")
    x = act["x"].view(torch.int16).numpy().view(np.uint16)
    logits = act["logits"].numpy()
    tokens = np.arange(n)
    ids, _ = O.route(logits[tokens], wl.k)
    need = [int(e) for e in np.unique(ids)]
    shp = {"g": (wl.E, wl.I, wl.H), "d": (wl.E, wl.H, wl.I)}
    drawn = {}

    def draw(e):
        drawn[e] = {n_: t.numpy() for n_, t in W.make_expert_weights(wl, e, seed, "cpu").items()}

    with cf.ThreadPoolExecutor(min(8, O.default_threads())) as ex:
        list(ex.map(draw, need))
    arrays = {}
    for key, name in (("g", "w_gate"), ("u", "w_up"), ("d", "w_down")):
        s = shp["d" if key == "d" else "g"]
        codes = np.zeros((s[0], s[1], s[2] // 2), np.uint8)  # untouched experts stay unallocated pages
        sf = np.zeros((s[0], s[1], s[2] // 16), np.uint8)
        sc = np.ones(s[0], np.float32)

        def one(e):
            c, f, t = O.quantize(drawn[e][name])
            codes[e], sf[e], sc[e] = c, f, t

        # ctypes releases the GIL while the oracle runs, so threads quantise in parallel
        with cf.ThreadPoolExecutor(O.default_threads()) as ex:
            list(ex.map(one, need))
        arrays[key] = (codes, sf, sc)
    s_x = np.float32(np.abs((x.astype(np.uint32) << 16).view(np.float32)).max()) / np.float32(2688)
    return x[tokens], logits[tokens], arrays, float(s_x)


def oracle_call(wl: W.Workload, inp, nthreads: int, a16: bool = False, shared=None):
    """One oracle pass over the sampled tokens (h scales calibrated by the oracle itself)."""
    import oracle as O
    x, logits, arr, s_x = inp
    if a16:
        O.moe_ffn_w4a16(x, logits, wl.k, arr["g"], arr["u"], arr["d"], nthreads=nthreads, shared=shared)
    else:
        O.moe_ffn(x, logits, wl.k, arr["g"], arr["u"], arr["d"], x_scale=s_x, h_scale=None, nthreads=nthreads,
                  shared=shared)


def oracle_rate(wl: W.Workload, budget_s: float, max_tokens: int, a16: bool = False, shared=None,
                nthreads: int | None = None, inp=None):
    """Tokens/s of the oracle on a bounded token sample of the workload (host cores)."""
    import oracle as O
    n = min(wl.T, max_tokens)
    inp = inp if inp is not None else oracle_inputs(wl, n)
    nth = nthreads or O.default_threads()
    done, t0 = 0, time.perf_counter()
    while True:
        oracle_call(wl, inp, nth, a16, shared)
        done += n
        el = time.perf_counter() - t0
        if el >= budget_s or done >= 64 * n:
            break
    return done / el, nth, f"{n} of {wl.T} tokens per pass, {done // n} passes, {el:.1f} s"


def gpu_launches_per_step(layer) -> int:
    # route, permute, amax pre-pass (dynamic x scale), quantise, gate/up, down, combine
    return 6 + (1 if layer.x_scale is None else 0)


# the default run: the headline workload first, then the other configurations
HEADLINE = "decode"
ALL_WORKLOADS = ("decode", "tiny", "prefill_chunk", "long_prefill", "dense", "dense_t1")
# workloads whose oracle is also timed on one host thread (small enough to finish in seconds)
SINGLE_THREAD = ("tiny", "decode", "dense_t1")


def workload_config(wl: W.Workload, world: int) -> dict:
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "top_k": wl.k,
            "zipf_s": wl.zipf_s, "outlier_frac": wl.outlier_frac,
            "l2": "flushed before every step (256 MiB write, then 256 MiB read)",
            "seed": 0, "parallelism": f"replicas x{world}"}


def measure(wl: W.Workload, args, dev, local: int, rank: int, world: int, dist_on: bool, cpu_budget: float,
            pk: dict) -> dict:
    """Times one workload on this rank's GPU (every rank takes the same collective steps) and,
    on rank 0 of a one-GPU run, the oracle on a bounded sample of it."""
    a16 = args.act == "bf16"
    path = {"auto": C.PATH_AUTO, "gemv": C.PATH_GEMV, "tcgen05": C.PATH_GEMM}[args.path]
    launch = {"auto": C.LAUNCH_AUTO, "single": C.LAUNCH_SINGLE, "multi": C.LAUNCH_MULTI,
              "single_tile": C.LAUNCH_SINGLE_TILE, "single_local": C.LAUNCH_SINGLE_LOCAL}[args.launch]
    single = launch in (C.LAUNCH_SINGLE, C.LAUNCH_SINGLE_TILE, C.LAUNCH_SINGLE_LOCAL)
    if single and not (wl.T <= 16 and path != C.PATH_GEMV and args.act == "nvfp4" and not args.shared_I
                       and (launch != C.LAUNCH_SINGLE_LOCAL or (wl.I % 256 == 0 and wl.I // 256 <= 63))):
        launch = C.LAUNCH_AUTO  # the single launch does not apply to this workload
    act, experts, layer = setup_layer(wl, dev, path=path, launch=launch)
    shared, shared_bits = None, None
    if args.shared_I:  # a BF16 shared expert, N(0, 1/sqrt(fan_in)) rounded to bf16
        gen = torch.Generator(device=dev).manual_seed(7)
        Is = args.shared_I
        sg = (torch.randn(Is, wl.H, generator=gen, device=dev) / wl.H ** 0.5).to(torch.bfloat16)
        su = (torch.randn(Is, wl.H, generator=gen, device=dev) / wl.H ** 0.5).to(torch.bfloat16)
        sd = (torch.randn(wl.H, Is, generator=gen, device=dev) / Is ** 0.5).to(torch.bfloat16)
        shared = (ops.shared_expert_w13(sg, su), sd)
        shared_bits = tuple(t.cpu().view(torch.int16).numpy().view(np.uint16) for t in (sg, su, sd))
    if a16:  # the same experts, weight-only
        layer = ops.MoeFFN(experts, wl.k, None, act=C.ACT_BF16, shared=shared)
    elif shared is not None:
        layer = ops.MoeFFN(experts, wl.k, layer.h_scale, path=path, shared=shared, launch=launch)
    flush = L2Flush(dev)
    with ClockSampler(local) as clk:
        step_ms, stage_ms, launches = time_steps(layer, act, args.steps, args.warmup, flush, dist_on)
    ms_per_step, value = job_throughput(max_over_ranks(sum(step_ms)), args.steps, world, wl.T)

    e2e_ms, h2d, d2h = time_e2e(layer, act, args.steps, args.warmup, flush)
    e2e_ms = max_over_ranks(e2e_ms)

    im = layer.intermediates(wl.T)
    n_active = int(im["active"][0].item())
    gemm_path = im["path"] == C.PATH_GEMM
    single = bool(layer.layout(wl.T).single_launch)
    alg = algorithmic(wl, n_active, gemm_path, a16, args.shared_I)
    # the dominant kernel (its stage is "gate_up"): the whole layer in one launch for batches of
    # at most 16 tokens on the tensor-core path; else, up to 64 tokens with H <= 2I, both GEMMs
    # in one fused launch; otherwise the gate/up GEMM
    fused = not single and gemm_path and wl.T <= 64 and wl.H <= 2 * wl.I
    dom_ms = stage_ms["gate_up"]
    dom_bytes = alg["layer_bytes"] if single else alg["gemms_bytes"] if fused else alg["gate_up_bytes"]
    dom_flops = alg["flops"] if (single or fused) else alg["gate_up_flops"]
    roof = roofline(dom_bytes, dom_flops, dom_ms, pk)
    kernel = ("single-launch layer: routing, x quantisation, tcgen05 gate/up + SwiGLU + requant, down, "
              "ordered combine" if single
              else "fused gate/up + down tcgen05 grouped GEMM (SwiGLU + requant, weighted slots)" if fused
              else "gate_up tcgen05 grouped GEMM + SwiGLU + requant" if gemm_path
              else "gate_up GEMV (bf16 x, NVFP4 weights) + SwiGLU" if a16
              else "gate_up GEMV + SwiGLU + requant")
    roof.update({"kernel": kernel,
                 "traffic": (measured_traffic(wl.name, "layer_fused.cu") if single
                             else measured_traffic(wl.name) if gemm_path else None),
                 "peak_source": pk["source"] + (f" ({pk['fp4_source']})" if roof["bound"] == "tensor" else ""),
                 "algorithmic_bytes_per_launch": dom_bytes,
                 "algorithmic_flops_per_launch": dom_flops, "touched_experts": n_active,
                 "launch_ms": dom_ms})
    layer_roof = roofline(alg["layer_bytes"], alg["flops"], ms_per_step, pk)
    layer_bw = alg["layer_bytes"] / (ms_per_step * 1e-3) / 1e9
    del layer, experts, act
    torch.cuda.empty_cache()
    if dist_on:
        torch.distributed.barrier()

    cpu = None
    if rank == 0 and world == 1 and cpu_budget > 0:
        n_cpu = min(wl.T, ORACLE_SAMPLE.get(wl.name, 4))
        inp = oracle_inputs(wl, n_cpu)
        v, cores, sample = oracle_rate(wl, cpu_budget, max_tokens=n_cpu, a16=a16, shared=shared_bits, inp=inp)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
               "sample": sample}
        if wl.name in SINGLE_THREAD:
            v1, _, s1 = oracle_rate(wl, min(cpu_budget, 4.0), max_tokens=n_cpu, a16=a16, shared=shared_bits,
                                    nthreads=1, inp=inp)
            cpu["single_thread"] = {"value": v1, "unit": "tokens/s", "cores": 1, "sample": s1}

    return {
        "value": value, "ms_per_step": ms_per_step, "config": workload_config(wl, world),
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": world * wl.T / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": (launches if launches is not None else 7) * args.steps,
        "launches_per_step": launches, "clocks": clk.summary(), "stages_ms": stage_ms,
        "layer": {"bytes": alg["layer_bytes"], "flops": alg["flops"], "hbm_gbs": layer_bw,
                  "hbm_frac": layer_bw / pk["hbm_gbs"], "hbm_frac_of_8tbs": layer_bw / NOMINAL_HBM_GBS,
                  "tflops": alg["flops"] / (ms_per_step * 1e-3) / 1e12,
                  "fp4_frac": alg["flops"] / (ms_per_step * 1e-3) / 1e12 / pk["fp4_tflops"],
                  "binding": layer_roof},
        "path": {C.PATH_GEMV: "gemv", C.PATH_GEMM: "tcgen05"}.get(im["path"], "?")
                + (" (single launch)" if single else ""),
    }


def compact(rec: dict) -> dict:
    """A workload's entry in the headline line's `workloads` object."""
    out = {k: rec[k] for k in ("value", "ms_per_step", "roofline", "e2e", "clocks", "stages_ms", "path",
                               "launches_per_step")}
    out["unit"] = "tokens/s"
    out["config"] = rec["config"]
    out["layer_binding"] = rec["layer"]["binding"]
    out["layer_bytes"] = rec["layer"]["bytes"]
    out["layer_flops"] = rec["layer"]["flops"]
    out["cpu_baseline"] = rec["cpu_baseline"]
    return out


def reference_arm(args, wl: W.Workload, rank: int, world: int, dist_on: bool):
    """The oracle on the host cores, on a bounded token sample of the workload per step.
    Inputs are drawn on the host (oracle_inputs): this arm never touches the GPU library."""
    if rank != 0:
        if dist_on:
            torch.distributed.destroy_process_group()
        return
    import oracle as O
    n = min(wl.T, ORACLE_SAMPLE.get(wl.name, 4))
    inp = oracle_inputs(wl, n)
    nth = O.default_threads()
    a16 = args.act == "bf16"
    for _ in range(args.warmup):
        oracle_call(wl, inp, nth, a16)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_call(wl, inp, nth, a16)
    el = time.perf_counter() - t0
    value = n * args.steps / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nth, "cpu_model": cpu_model(),
                             "kind": "oracle", "sample": f"{n} of {wl.T} tokens per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="all", choices=["all"] + sorted(W.WORKLOADS),
                    help="all: the headline decode workload, then every other configuration (default)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle time for the headline's cpu_baseline (a third of it per other workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", default="auto", choices=["auto", "gemv", "tcgen05"],
                    help="layer path: auto, the GEMV path or the tcgen05 grouped GEMM")
    ap.add_argument("--act", default="nvfp4", choices=["nvfp4", "bf16"],
                    help="activations: nvfp4 (W4A4) or bf16 (the weight-only W4A16 variant, GEMV path)")
    ap.add_argument("--shared-I", type=int, default=0,
                    help="add a BF16 shared expert of this intermediate size (0: none)")
    ap.add_argument("--launch", default="auto", choices=["auto", "single", "multi", "single_tile", "single_local"],
                    help="batches of at most 16 tokens: one persistent launch (its schedule chosen per call, or "
                         "forced tile-level / expert-local), the multi-launch path, or automatic")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    names = ALL_WORKLOADS if args.workload == "all" else (args.workload,)

    if args.impl == "reference":
        if dist_on:
            import datetime
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
        reference_arm(args, W.WORKLOADS[names[0]], rank, world, dist_on)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    pk = peaks(dev)
    recs = {}
    for i, name in enumerate(names):
        budget = 0.0 if args.no_cpu_baseline else (args.cpu_budget if i == 0 else args.cpu_budget / 3)
        recs[name] = measure(W.WORKLOADS[name], args, dev, local, rank, world, dist_on, budget, pk)

    if rank == 0:
        head = recs[names[0]]
        a16 = args.act == "bf16"
        cfg = dict(head["config"])
        if a16:
            cfg["act"] = "w4a16 (bf16 activations, NVFP4 weights)"
        if args.shared_I:
            cfg["shared_expert"] = f"bf16 SwiGLU, I_s={args.shared_I}"
        line = {
            "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 x nvfp4 (w4a16, fp32 accumulate)" if a16 else "nvfp4 (e2m1 x e4m3, fp32 accumulate)",
            "data": "synthetic", "config": cfg, "roofline": head["roofline"], "cpu_baseline": head["cpu_baseline"],
            "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"], "launches_per_step": head["launches_per_step"],
            "timing": "CUDA-graph replay of the layer's forward, events on the replay stream",
            "clocks": head["clocks"], "stages_ms": head["stages_ms"], "layer": head["layer"], "path": head["path"],
            "peaks": {k: pk[k] for k in ("hbm_gbs", "bf16_tflops", "fp4_tflops", "source", "fp4_source")},
        }
        if len(names) > 1:
            line["workloads"] = {n: compact(r) for n, r in recs.items()}
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
