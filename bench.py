"""Benchmark of the BitLinear forward on B200: one JSON line on rank 0.

Headline workload (the decode metric is quoted on it): the 3B-class decode
GEMV pair K=3200 -> N=8640 and K=8640 -> N=3200 at M=1 token, bf16
activations and outputs, latent weights N(0, 0.02^2) packed to 2 bits.
One step = for each of the two matrices, per-token absmax quantisation
plus integer accumulation and rescale (the per-token half of the layer;
packing is load-time and is timed separately under "pack").  Inputs are
resident in HBM; the packed weights rotate through enough copies that each
step reads them from HBM, not L2.  ``value`` = algorithmic bytes of the
step / device time, in GB/s.

Also reported on the same line: "prefill" (7B-class M=2048 GEMM on the
tensor cores, int8 TOPS vs the int8 peak), "pack" (load-time), "roofline"
of the dominant kernel, "e2e" through the public API with host buffers,
"cpu_baseline" (the CPU oracle on the host cores, rank 0 only) and the SM
clocks seen during the timed region.

--impl reference times the CPU oracle on the same workload (the method's
reference implementation here), each step a bounded sample of it.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import ctypes  # noqa: E402

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

METRIC = "BitLinear decode GB/s & %HBM roofline (M=1); prefill int8 TOPS & %peak"
WORKLOAD = "decode_3b"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 : 2.25 PFLOP/s bf16)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def linear_bytes(M, K, N, out_bytes=2, in_bytes=2):
    """Algorithmic bytes of the fused per-token layer on one matrix: read the
    packed weights (N*ceil(K/4)), the activations (M*K*in) and gamma (4),
    write y (M*N*out).  x~, eta and xsum never leave the chip."""
    return N * ((K + 3) // 4) + M * K * in_bytes + 4 + M * N * out_bytes


# ----------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(v, world):
    if world == 1:
        return v
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        dist.barrier()


# ----------------------------------------------------------------- clocks

CLOCK_Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
           "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
           "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index, log_dir=None):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(log_dir or tempfile.gettempdir(),
                                 "clocks_bench_%d.csv" % os.getpid())

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + CLOCK_Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "samples": len(rows), "reasons": reasons}


# ----------------------------------------------------------------- our arm

class Capture:
    """CUDA graph of a list of C-ABI calls, replayed for timing.  replay()
    launches on the current stream: callers time it inside timed(), which
    makes the timed stream current."""

    def __init__(self, calls, stream):
        self.graph = torch.cuda.CUDAGraph()
        self.stream = stream
        with torch.cuda.stream(stream):
            with torch.cuda.graph(self.graph, stream=stream):
                for fn in calls:
                    fn()

    def replay(self):
        assert torch.cuda.current_stream() == self.stream, "replay on the timed stream"
        self.graph.replay()


def timed(fn_replays, stream, world):
    """Device time of fn_replays(): events recorded on `stream`, and the work
    (graph replays, library calls) issued on that same stream.  A short sleep
    kernel ahead of the start event keeps the stream busy while the host
    enqueues the work, so no host-submission gap falls inside a short timed
    region."""
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(200000)  # about 0.1 ms, before the start event
        t0.record(stream)
        fn_replays()
        t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return t0.elapsed_time(t1) / 1e3  # seconds


def run_ours(args, world, rank, local):
    from ternary_weight_linear_04_b200 import _lib, build as libbuild, inputs
    from ternary_weight_linear_04_b200 import bitlinear as bl

    if rank == 0 or world == 1:
        libbuild.build()
    barrier(world)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    L = _lib.lib()
    stream = torch.cuda.Stream(device=dev)
    sptr = ctypes.c_void_p(stream.cuda_stream)
    peaks, peak_src = load_peaks()
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20

    wl = inputs.WORKLOADS[WORKLOAD]
    M = args.m
    mats = []
    for j, mat in enumerate(wl.matrices):
        W, x = inputs.make_matrix_inputs(wl, j, m_max=max(M, 64))  # 64 rows for the M sweep
        Wd = torch.from_numpy(W).to(dev)
        with torch.cuda.stream(stream):
            packed, gamma = bl.pack_weights(Wd, stream=stream)
        x_all = torch.from_numpy(x).to(dev).to(torch.bfloat16)
        xd = x_all[:M]
        mats.append(dict(K=mat.K, N=mat.N, W=Wd, packed=packed, gamma=gamma, x=xd, x_all=x_all,
                         xq=torch.empty((M, mat.K), dtype=torch.int8, device=dev),
                         eta=torch.empty(M, dtype=torch.float32, device=dev),
                         xsum=torch.empty(M, dtype=torch.int32, device=dev),
                         y=torch.empty((M, mat.N), dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()
    step_w_bytes = sum(m["N"] * ((m["K"] + 3) // 4) for m in mats)
    copies = max(2, int(np.ceil(3 * l2 / step_w_bytes)))
    for m in mats:
        m["copies"] = [(m["packed"], m["gamma"])] + [(m["packed"].clone(), m["gamma"].clone())
                                                     for _ in range(copies - 1)]
    torch.cuda.synchronize()

    P = ctypes.c_void_p

    def linear_call(m, c):
        """One call of the whole per-token layer (bitlinear_linear): quantise,
        accumulate, rescale; weights packed at load time are static."""
        pk, g = m["copies"][c]
        args_ = (P(m["x"].data_ptr()), _lib.BL_BF16, M, m["K"], P(pk.data_ptr()), P(g.data_ptr()),
                 m["N"], P(m["y"].data_ptr()), _lib.BL_BF16, P(m["xq"].data_ptr()),
                 P(m["eta"].data_ptr()), P(m["xsum"].data_ptr()), None,
                 _lib.BL_FLAG_WEIGHTS_STATIC, sptr)
        return lambda: _chk(L.bitlinear_linear(*args_), "linear")

    def step_calls(c):
        return [linear_call(m, c) for m in mats]

    # Warm-up (also sets kernel attributes outside capture).
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            for fn in step_calls(i % copies):
                fn()
    torch.cuda.synchronize()

    G = copies  # one graph walks every weight copy once
    full, rem = divmod(args.steps, G)
    g_full = Capture([fn for c in range(G) for fn in step_calls(c)], stream)
    g_rem = Capture([fn for c in range(rem) for fn in step_calls(c)], stream) if rem else None
    # graph warm-up (both graphs: a graph's first replay uploads it)
    with torch.cuda.stream(stream):
        for _ in range(2):
            g_full.replay()
            if g_rem:
                g_rem.replay()
    torch.cuda.synchronize()

    def replays():
        for _ in range(full):
            g_full.replay()
        if g_rem:
            g_rem.replay()

    # The timed window (exactly --steps steps) is repeated: at least 5 times
    # and until 50 ms of device time; the line reports the median window.
    # The window count is derived from the first window's max over ranks, so
    # every rank runs the same number of windows.
    with ClockSampler(local, args.clocks_dir) as clk:
        t_first = max_over_ranks(timed(replays, stream, world), world)
        n_win = min(2000, max(5, int(np.ceil(0.05 / max(t_first, 1e-9)))))
        if args.windows:
            n_win = args.windows
        wins = [t_first] + [max_over_ranks(timed(replays, stream, world), world)
                            for _ in range(n_win - 1)]
    t_step = statistics.median(wins)
    per_step_bytes = sum(linear_bytes(M, m["K"], m["N"]) for m in mats)
    value = world * per_step_bytes * args.steps / t_step / 1e9
    launches = len(mats) * args.steps  # one fused decode kernel per matrix

    # The step is nothing but the dominant kernel (k_decode, one launch per
    # matrix), so its per-launch time is the timed region / launches.
    avg_launch = t_step / launches
    bytes_per_launch = per_step_bytes / len(mats)
    achieved = bytes_per_launch / avg_launch / 1e9
    hbm_peak = float(peaks["hbm_gbs"])
    paths = [bl.select_path(M, m["K"], m["N"], m["xq"], m["copies"][0][0], m["y"]) for m in mats]
    # which fused decode kernel bitlinear_linear runs for each matrix
    sms = props.multi_processor_count
    reg_shapes = [bl.decode_reg_shape(m["K"], m["N"], sms) if M == 1 else None for m in mats]
    kernel = "k_decode_reg" if all(reg_shapes) else "k_decode"
    roofline = {"kernel": "%s (fused quantise + accumulate + rescale)" % kernel,
                "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "traffic": load_traffic(kernel),
                "shapes": reg_shapes if kernel == "k_decode_reg" else None,
                "peak_source": peak_src + " hbm_gbs (burst copy)",
                "avg_launch_us": round(avg_launch * 1e6, 3),
                "algorithmic_bytes_per_launch": bytes_per_launch}

    out = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(t_step / args.steps * 1e3, 6), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "int8",
           "data": "synthetic (seeded N(0,0.02^2) latent weights, N(0,1) bf16 activations)",
           "config": {"workload": "decode_3b: K=3200->N=8640 and K=8640->N=3200, M=%d, bf16 in/out"
                                  % M,
                      "M": M, "parallelism": "replicas" if world > 1 else "single GPU",
                      "l2": "inputs larger than L2: %d rotating packed-weight copies (%.0f MB > 3x L2)"
                            % (copies, copies * step_w_bytes / 1e6),
                      "paths": paths},
           "windows": {"n": n_win, "steps_each": args.steps,
                       "median_ms_per_step": round(t_step / args.steps * 1e3, 6),
                       "min_ms_per_step": round(min(wins) / args.steps * 1e3, 6),
                       "max_ms_per_step": round(max(wins) / args.steps * 1e3, 6)},
           "roofline": roofline, "gpu_launches": launches,
           "clocks": clk.summary()}

    sections = (set(args.sections.split(",")) if args.sections else
                {"e2e", "prefill", "pack", "sweep", "layer70b", "crossover", "base3", "rmsnorm"})
    if args.quick:
        sections = set()
    if "e2e" in sections:
        out["e2e"] = run_e2e(args, mats, M, stream, world)
    if "prefill" in sections:
        out["prefill"] = run_prefill(args, dev, stream, peaks, peak_src, world, l2)
    if "pack" in sections:
        out["pack"] = run_pack(mats, stream, world)
    if "sweep" in sections:
        out["decode_sweep"] = run_sweep(mats, stream, world, peaks)
    if "layer70b" in sections or "crossover" in sections:
        for m in mats:  # free the headline workload's copies first
            m["copies"] = m["copies"][:1]
        torch.cuda.empty_cache()
    if "layer70b" in sections:
        out["layer_70b"] = run_layer70b(dev, stream, world, peaks, l2)
    if "crossover" in sections:
        out["crossover"] = run_crossover(dev, stream, world, peaks, l2)
    if "base3" in sections:
        out["base3"] = run_base3(dev, stream, world, peaks, l2)
    if "rmsnorm" in sections:
        out["rmsnorm"] = run_rmsnorm(dev, stream, world, peaks, l2)
    if (rank == 0) and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = run_cpu_baseline(args.cpu_seconds)
    return out


def _chk(status, what):
    if status != 0:
        raise RuntimeError("%s failed with status %d" % (what, status))


def load_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary
    (profiles/traffic.md, a markdown table), or None if absent."""
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p):
        return None
    for line in open(p):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 2 and cells[0] == kernel:
            try:
                return int(cells[1])
            except ValueError:
                return None
    return None


def run_e2e(args, mats, M, stream, world):
    """Through the public Python API, host buffers in, host buffers out.

    Each step copies that step's x from pinned host memory to the device,
    runs bitlinear.linear on both matrices and copies y back to pinned host
    memory, then synchronises the stream.  As a decode loop runs it, the
    step's calls are captured once in a CUDA graph per rotated weight copy
    and replayed; the same step issued eagerly from Python is timed too
    ("eager")."""
    from ternary_weight_linear_04_b200 import bitlinear as bl
    xs_h = [m["x"].cpu().pin_memory() for m in mats]
    ys_h = [torch.empty_like(m["y"], device="cpu").pin_memory() for m in mats]
    # The graph's step: every matrix's x in one pinned staging buffer, one
    # copy in; every y into one device buffer, one copy out.
    x_sizes = [m["x"].numel() for m in mats]
    y_sizes = [m["y"].numel() for m in mats]
    xcat_h = torch.cat([x.flatten() for x in xs_h]).pin_memory()
    ycat_h = torch.empty(sum(y_sizes), dtype=mats[0]["y"].dtype).pin_memory()
    xcat_d = torch.empty_like(xcat_h, device=mats[0]["x"].device)
    ycat_d = torch.empty_like(ycat_h, device=mats[0]["y"].device)
    xs_d = [v.view(m["x"].shape) for v, m in zip(torch.split(xcat_d, x_sizes), mats)]
    ys_d = [v.view(m["y"].shape) for v, m in zip(torch.split(ycat_d, y_sizes), mats)]
    steps = max(3, min(args.steps, 500))
    copies = len(mats[0]["copies"])

    def calls(i):
        xcat_d.copy_(xcat_h, non_blocking=True)
        for j, m in enumerate(mats):
            pk, g = m["copies"][i % copies]
            bl.linear(xs_d[j], pk, g, m["N"], out_dtype=torch.bfloat16, weights_static=True,
                      stream=stream, out=ys_d[j])
        ycat_h.copy_(ycat_d, non_blocking=True)

    def eager(i):
        for j, m in enumerate(mats):
            pk, g = m["copies"][i % copies]
            xd = xs_h[j].to(m["x"].device, non_blocking=True)
            y = bl.linear(xd, pk, g, m["N"], out_dtype=torch.bfloat16, weights_static=True,
                          stream=stream)
            ys_h[j].copy_(y, non_blocking=True)
        stream.synchronize()

    with torch.cuda.stream(stream):
        for i in range(copies):
            calls(i)
        stream.synchronize()
        graphs = []
        for i in range(copies):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                calls(i)
            graphs.append(gr)
        for i in range(3):
            graphs[i % copies].replay()
            stream.synchronize()
        barrier(world)
        t0 = time.perf_counter()
        for i in range(steps):
            graphs[i % copies].replay()
            stream.synchronize()
        t = time.perf_counter() - t0
        for i in range(3):
            eager(i)
        t1 = time.perf_counter()
        for i in range(steps):
            eager(i)
        te = time.perf_counter() - t1
    del graphs
    t = max_over_ranks(t, world)
    te = max_over_ranks(te, world)
    b = sum(linear_bytes(M, m["K"], m["N"]) for m in mats)
    h2d = sum(M * m["K"] * 2 for m in mats)
    d2h = sum(M * m["N"] * 2 for m in mats)
    return {"value": round(world * b * steps / t / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(t / steps * 1e3, 4), "steps": steps,
            "note": "public API (bitlinear.linear) per matrix; the step's inputs in one pinned "
                    "host buffer, one copy in, the outputs copied out in one; captured in a CUDA "
                    "graph and replayed every step; stream synchronised every step",
            "eager": {"value": round(world * b * steps / te / 1e9, 2),
                      "ms_per_step": round(te / steps * 1e3, 4),
                      "note": "the same step issued from Python every time"}}


def run_prefill(args, dev, stream, peaks, peak_src, world, l2):
    """7B-class prefill: M=2048, K=4096, N=11008 on the tcgen05 path.  The
    packed weights, x, x~ and y rotate through enough copies (> 3x L2) that
    every forward reads its inputs from HBM.  Reported twice: the
    accumulate kernel alone (x~ given) and the whole layer (quantiser +
    accumulate)."""
    from ternary_weight_linear_04_b200 import inputs
    from ternary_weight_linear_04_b200 import bitlinear as bl
    wl = inputs.WORKLOADS["prefill_7b"]
    W, x = inputs.make_matrix_inputs(wl, 0)
    M, K, N = x.shape[0], W.shape[1], W.shape[0]
    with torch.cuda.stream(stream):
        packed, gamma = bl.pack_weights(torch.from_numpy(W).to(dev), stream=stream)
    xd0 = torch.from_numpy(x).to(dev).to(torch.bfloat16)
    torch.cuda.synchronize()
    set_bytes = packed.numel() + M * K * 3 + M * N * 2  # packed W, x (bf16) + x~, y
    copies = max(2, int(np.ceil(3 * l2 / set_bytes)))
    sets = []
    for _ in range(copies):
        xd = xd0.clone()
        with torch.cuda.stream(stream):
            xq, eta, xsum = bl.quant_act(xd, stream=stream)
        sets.append(dict(packed=packed.clone(), gamma=gamma.clone(), x=xd, xq=xq, eta=eta, xsum=xsum,
                         y=torch.empty((M, N), dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()
    path = bl.select_path(M, K, N, sets[0]["xq"], packed, sets[0]["y"])

    def fwd(c):
        return lambda: bl.forward(c["xq"], c["eta"], c["xsum"], c["packed"], c["gamma"], N,
                                  stream=stream, out=c["y"], weights_static=True)

    def quant(c):
        return lambda: bl.quant_act(c["x"], stream=stream, out=(c["xq"], c["eta"], c["xsum"]))

    def timed_calls(calls, reps):
        with torch.cuda.stream(stream):
            for fn in calls:
                fn()
        torch.cuda.synchronize()
        g = Capture(calls, stream)
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        ts = [max_over_ranks(timed(lambda: [g.replay() for _ in range(reps)], stream, world), world)
              for _ in range(5)]
        return statistics.median(ts) / (reps * copies)

    per = timed_calls([fwd(c) for c in sets], 10)
    tq = timed_calls([quant(c) for c in sets], 10)
    layer = timed_calls([f for c in sets for f in (quant(c), fwd(c))], 10)
    ops = 2.0 * M * N * K
    peak = float(peaks["bf16_tflops"]) * INT8_PER_BF16
    qbytes = M * K * 3 + 8 * M
    del sets
    torch.cuda.empty_cache()
    return {"workload": "prefill_7b: M=2048, K=4096, N=11008, bf16 in/out", "path": path,
            "kernel": "k_gemm_tc", "us_per_forward": round(per * 1e6, 2),
            "tops": round(ops / per / 1e12, 1), "int8_peak_tops": round(peak, 1),
            "frac": round(ops / per / 1e12 / peak, 4), "bound": "tensor",
            "traffic": load_traffic("k_gemm_tc"),
            "peak_source": "%s bf16_tflops (burst) x %.0f nominal int8:bf16 ratio" % (peak_src, INT8_PER_BF16),
            "inputs": "%d rotating sets of packed W, x, x~ and y (%.0f MB > 3x L2)"
                      % (copies, copies * set_bytes / 1e6),
            "addsub_ops_needed_frac": "nnz(W~)/(N*K) of the dense ops (about 0.69)",
            "quant_us": round(tq * 1e6, 2), "quant_gbs": round(qbytes / tq / 1e9, 1),
            "layer_us": round(layer * 1e6, 2), "layer_tops": round(ops / layer / 1e12, 1),
            "layer_frac": round(ops / layer / 1e12 / peak, 4)}


def time_linear_step(mats, M, stream, world, min_seconds=0.25, xkey="x", groups=None):
    """Seconds per step of one bitlinear_linear call per matrix (static
    weights), CUDA graph over every rotating packed copy, max over ranks.
    mats: dicts with K, N, copies [(packed, gamma)], m[xkey] (>= M rows, bf16).
    groups: lists of matrix indices sharing one input, each run as one
    bitlinear_linear_group call (the others one call each)."""
    from ternary_weight_linear_04_b200 import _lib
    L = _lib.lib()
    P = ctypes.c_void_p
    dev = mats[0][xkey].device
    sptr = ctypes.c_void_p(stream.cuda_stream)
    bufs = []
    for m in mats:
        bufs.append(dict(x=m[xkey][:M].contiguous(),
                         y=torch.empty((M, m["N"]), dtype=torch.bfloat16, device=dev),
                         xq=torch.empty((M, m["K"]), dtype=torch.int8, device=dev),
                         eta=torch.empty(M, dtype=torch.float32, device=dev),
                         xsum=torch.empty(M, dtype=torch.int32, device=dev)))

    def call(m, b, c):
        pk, g = m["copies"][c]
        a = (P(b["x"].data_ptr()), _lib.BL_BF16, M, m["K"], P(pk.data_ptr()), P(g.data_ptr()), m["N"],
             P(b["y"].data_ptr()), _lib.BL_BF16, P(b["xq"].data_ptr()), P(b["eta"].data_ptr()),
             P(b["xsum"].data_ptr()), None, _lib.BL_FLAG_WEIGHTS_STATIC, sptr)
        return lambda: _chk(L.bitlinear_linear(*a), "linear")

    def call_group(idx, c):
        n = len(idx)
        arr = ctypes.c_void_p * n
        pk = arr(*[P(mats[i]["copies"][c][0].data_ptr()) for i in idx])
        gm = arr(*[P(mats[i]["copies"][c][1].data_ptr()) for i in idx])
        ns = (ctypes.c_int64 * n)(*[mats[i]["N"] for i in idx])
        ys = arr(*[P(bufs[i]["y"].data_ptr()) for i in idx])
        b0 = bufs[idx[0]]
        a = (P(b0["x"].data_ptr()), _lib.BL_BF16, M, mats[idx[0]]["K"], n, pk, gm, ns, ys,
             _lib.BL_BF16, _lib.BL_FLAG_WEIGHTS_STATIC, sptr)
        keep = (pk, gm, ns, ys)
        return lambda: (_chk(L.bitlinear_linear_group(*a), "linear_group"), keep)

    copies = len(mats[0]["copies"])
    if groups is None:
        calls = [call(m, b, c) for c in range(copies) for m, b in zip(mats, bufs)]
    else:
        grouped = {i for g in groups for i in g}
        calls = []
        for c in range(copies):
            for i, (m, b) in enumerate(zip(mats, bufs)):
                g = next((g for g in groups if g[0] == i), None)
                if g is not None:
                    calls.append(call_group(g, c))
                elif i not in grouped:
                    calls.append(call(m, b, c))
    with torch.cuda.stream(stream):
        for fn in calls:
            fn()
    torch.cuda.synchronize()
    g = Capture(calls, stream)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    t1 = timed(lambda: g.replay(), stream, world)
    reps = max(3, int(min_seconds / max(t1, 1e-6)))
    t = timed(lambda: [g.replay() for _ in range(reps)], stream, world)
    t = max_over_ranks(t, world)
    return t / (reps * copies)


def make_bench_mats(wl_name, M, dev, stream, l2, copies=None):
    """Packed matrices of a workload (+ rotating copies past 3x L2) and its
    activations (M rows)."""
    from ternary_weight_linear_04_b200 import inputs
    from ternary_weight_linear_04_b200 import bitlinear as bl
    wl = inputs.WORKLOADS[wl_name]
    mats = []
    for j, mat in enumerate(wl.matrices):
        W, x = inputs.make_matrix_inputs(wl, j, m_max=M)
        with torch.cuda.stream(stream):
            Wd = torch.from_numpy(W).to(dev)
            packed, gamma = bl.pack_weights(Wd, stream=stream)
        torch.cuda.synchronize()
        del Wd, W
        mats.append(dict(K=mat.K, N=mat.N, name=mat.name, packed=packed, gamma=gamma,
                         x=torch.from_numpy(x).to(dev).to(torch.bfloat16)))
    wbytes = sum(m["N"] * ((m["K"] + 3) // 4) for m in mats)
    if copies is None:
        copies = max(2, int(np.ceil(3 * l2 / wbytes)))
    for m in mats:
        m["copies"] = [(m["packed"], m["gamma"])] + [(m["packed"].clone(), m["gamma"].clone())
                                                     for _ in range(copies - 1)]
    torch.cuda.synchronize()
    return mats, copies, wbytes


def layer_kernels(M, m):
    """The kernels bitlinear_linear launches for a bf16 layer of M tokens on
    the matrix m, from the library's own shape queries."""
    from ternary_weight_linear_04_b200 import bitlinear as bl
    K, N = m["K"], m["N"]
    if M == 1 and bl.decode_reg_shape(K, N) is not None:
        return "k_decode_reg (fused)"
    if M == 2 and bl.decode_regm_shape(M, K, N) is not None:
        return "k_decode_regm (fused)"
    if M <= 2 and bl.fused_decode_ok(M, K):
        return "k_decode (fused)"
    if M <= 8 and bl.decode_regm_shape(M, K, N) is not None:
        return "k_quant_bf16 + k_decode_regm"
    if M <= 16 and bl.decode_mma_shape(M, K, N) is not None:
        return "k_quant_bf16 + k_decode_mma"
    if bl.select_path(M, K, N, m["x_all"], m["packed"], m["x_all"]) == "gemv":
        return "k_quant_bf16 + k_decode"
    return "k_quant_bf16 + k_gemm_tc"


def run_sweep(mats, stream, world, peaks, Ms=(2, 4, 8, 12, 16, 32, 64)):
    """decode_3b at the other batch sizes: GB/s against HBM."""
    from ternary_weight_linear_04_b200 import bitlinear as bl
    hbm = float(peaks["hbm_gbs"])
    rows = []
    for M in Ms:
        t = time_linear_step(mats, M, stream, world, xkey="x_all")
        b = sum(linear_bytes(M, m["K"], m["N"]) for m in mats)
        paths = [layer_kernels(M, m) for m in mats]
        rows.append({"M": M, "us_per_step": round(t * 1e6, 2), "gbs": round(b / t / 1e9, 1),
                     "frac": round(b / t / 1e9 / hbm, 4), "paths": paths})
    return {"workload": "decode_3b: K=3200->N=8640 and K=8640->N=3200, bf16 in/out",
            "step": "one bitlinear_linear per matrix (quantise + accumulate + rescale)",
            "rows": rows}


def run_layer70b(dev, stream, world, peaks, l2):
    """One 70B-class decoder layer's 7 projections as 7 calls, M = 1 and 32."""
    hbm = float(peaks["hbm_gbs"])
    mats, copies, wbytes = make_bench_mats("layer_70b", 32, dev, stream, l2)
    rows = []
    for M in (1, 32):
        t = time_linear_step(mats, M, stream, world)
        b = sum(linear_bytes(M, m["K"], m["N"]) for m in mats)
        rows.append({"M": M, "us_per_layer": round(t * 1e6, 2), "gbs": round(b / t / 1e9, 1),
                     "frac": round(b / t / 1e9 / hbm, 4), "launches": 7 if M <= 4 else 14})
    # shared-input fusion: Wq|Wk|Wv and gate|up each as one grouped launch
    t = time_linear_step(mats, 1, stream, world, groups=[[0, 1, 2], [4, 5]])
    b = sum(linear_bytes(1, m["K"], m["N"]) for m in mats)
    rows.append({"M": 1, "grouped": "Wq|Wk|Wv and gate|up (bitlinear_linear_group)",
                 "us_per_layer": round(t * 1e6, 2), "gbs": round(b / t / 1e9, 1),
                 "frac": round(b / t / 1e9 / hbm, 4), "launches": 4})
    del mats
    torch.cuda.empty_cache()
    return {"workload": "layer_70b: Wq 8192^2, Wk/Wv 8192x1024, Wo 8192^2, gate/up 8192x28672, "
                        "down 28672x8192; 7 bitlinear_linear calls per step",
            "packed_bytes_per_layer": wbytes, "copies": copies, "rows": rows}


def run_crossover(dev, stream, world, peaks, l2):
    """8192x28672, Laplace weights, Student-t(3) activations with 1% x50
    outlier channels: both accumulate paths across M; the crossover is the
    smallest M at which the tensor-core path is the faster one."""
    from ternary_weight_linear_04_b200 import _lib
    from ternary_weight_linear_04_b200 import bitlinear as bl
    mats, copies, wbytes = make_bench_mats("outlier_sweep", 2048, dev, stream, l2)
    m = mats[0]
    K, N = m["K"], m["N"]
    hbm = float(peaks["hbm_gbs"])
    peak_t = float(peaks["bf16_tflops"]) * INT8_PER_BF16
    L = _lib.lib()
    P = ctypes.c_void_p
    sptr = ctypes.c_void_p(stream.cuda_stream)
    rows, cross = [], None
    for M in (1, 2, 4, 8, 64, 256, 2048):
        xq, eta, xsum = bl.quant_act(m["x"][:M].contiguous(), stream=stream)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        row = {"M": M}
        for path in (("gemv", "tcgen05") if M <= 4 else ("tcgen05",)):
            calls = []
            for c in range(copies):
                pk, g = m["copies"][c]
                a = (P(xq.data_ptr()), P(eta.data_ptr()), P(xsum.data_ptr()), M, K, P(pk.data_ptr()),
                     P(g.data_ptr()), N, P(y.data_ptr()), _lib.BL_BF16, None, bl.PATHS[path],
                     _lib.BL_FLAG_WEIGHTS_STATIC, sptr)
                calls.append(lambda a=a: _chk(L.bitlinear_forward_path(*a), path))
            with torch.cuda.stream(stream):
                for fn in calls:
                    fn()
            torch.cuda.synchronize()
            gr = Capture(calls, stream)
            with torch.cuda.stream(stream):
                gr.replay()
            torch.cuda.synchronize()
            reps = 20 if M <= 256 else 3
            t = max_over_ranks(timed(lambda: [gr.replay() for _ in range(reps)], stream, world),
                               world) / (reps * copies)
            b = linear_bytes(M, K, N, in_bytes=1)
            row[path] = {"us": round(t * 1e6, 2), "gbs": round(b / t / 1e9, 1),
                         "hbm_frac": round(b / t / 1e9 / hbm, 4),
                         "tops": round(2.0 * M * N * K / t / 1e12, 1),
                         "tensor_frac": round(2.0 * M * N * K / t / 1e12 / peak_t, 4)}
        if cross is None and "gemv" in row and row["tcgen05"]["us"] <= row["gemv"]["us"]:
            cross = M
        rows.append(row)
    del mats
    torch.cuda.empty_cache()
    return {"workload": "outlier_sweep: K=8192, N=28672, Laplace(0,0.02) W, Student-t(3) x with "
                        "1%% x50 channels; accumulate kernel only (x~ given)",
            "rows": rows,
            "crossover_M": cross if cross is not None else "above 4 (the CUDA-core decode path "
                                                           "takes M <= 4 and is faster there)"}


def run_base3(dev, stream, world, peaks, l2):
    """Base-3 packing (five trits per byte) against the 2-bit codes, x~ given,
    M = 1: the accumulate kernels on decode_3b and on 8192x28672."""
    from ternary_weight_linear_04_b200 import _lib, inputs
    from ternary_weight_linear_04_b200 import bitlinear as bl
    L = _lib.lib()
    P = ctypes.c_void_p
    sptr = ctypes.c_void_p(stream.cuda_stream)
    hbm = float(peaks["hbm_gbs"])
    rows = []
    for wl_name in ("decode_3b", "outlier_sweep"):
        wl = inputs.WORKLOADS[wl_name]
        mats = []
        for j, mat in enumerate(wl.matrices):
            W, x = inputs.make_matrix_inputs(wl, j, m_max=1)
            with torch.cuda.stream(stream):
                Wd = torch.from_numpy(W).to(dev)
                p2, g = bl.pack_weights(Wd, stream=stream)
                p3, _ = bl.pack_weights3(Wd, stream=stream)
                xq, eta, xsum = bl.quant_act(torch.from_numpy(x).to(dev).to(torch.bfloat16), stream=stream)
            torch.cuda.synchronize()
            del Wd, W
            mats.append(dict(K=mat.K, N=mat.N, p2=p2, p3=p3, g=g, xq=xq, eta=eta, xsum=xsum,
                             y=torch.empty((1, mat.N), dtype=torch.bfloat16, device=dev)))
        b2 = sum(m["N"] * ((m["K"] + 3) // 4) for m in mats)
        b3 = sum(m["p3"].numel() for m in mats)
        copies = max(2, int(np.ceil(3 * l2 / b3)))
        for m in mats:
            m["c2"] = [m["p2"]] + [m["p2"].clone() for _ in range(copies - 1)]
            m["c3"] = [m["p3"]] + [m["p3"].clone() for _ in range(copies - 1)]
        torch.cuda.synchronize()
        res = {"workload": wl_name, "packed_bytes_2bit": b2, "packed_bytes_base3": b3}
        for fmt in ("2bit", "base3"):
            calls = []
            for c in range(copies):
                for m in mats:
                    if fmt == "2bit":
                        a = (P(m["xq"].data_ptr()), P(m["eta"].data_ptr()), P(m["xsum"].data_ptr()), 1,
                             m["K"], P(m["c2"][c].data_ptr()), P(m["g"].data_ptr()), m["N"],
                             P(m["y"].data_ptr()), _lib.BL_BF16, None, _lib.BL_PATH_GEMV,
                             _lib.BL_FLAG_WEIGHTS_STATIC, sptr)
                        calls.append(lambda a=a: _chk(L.bitlinear_forward_path(*a), "forward"))
                    else:
                        a = (P(m["xq"].data_ptr()), P(m["eta"].data_ptr()), P(m["xsum"].data_ptr()), 1,
                             m["K"], P(m["c3"][c].data_ptr()), P(m["g"].data_ptr()), m["N"],
                             P(m["y"].data_ptr()), _lib.BL_BF16, None, sptr)
                        calls.append(lambda a=a: _chk(L.bitlinear_forward3(*a), "forward3"))
            with torch.cuda.stream(stream):
                for fn in calls:
                    fn()
            torch.cuda.synchronize()
            gr = Capture(calls, stream)
            with torch.cuda.stream(stream):
                gr.replay()
            torch.cuda.synchronize()
            reps = 20
            t = max_over_ranks(timed(lambda: [gr.replay() for _ in range(reps)], stream, world),
                               world) / (reps * copies)
            wb = b2 if fmt == "2bit" else b3
            res[fmt] = {"us_per_step": round(t * 1e6, 2), "weight_gbs": round(wb / t / 1e9, 1),
                        "hbm_frac": round(wb / t / 1e9 / hbm, 4),
                        "trits_per_ns": round(sum(m["N"] * m["K"] for m in mats) / t / 1e9, 1)}
        rows.append(res)
        del mats
        torch.cuda.empty_cache()
    return {"what": "accumulate kernels only (x~ given), M=1: bitlinear_forward (2-bit codes, "
                    "decode kernel) against bitlinear_forward3 (base-3, five trits per byte)",
            "rows": rows}


def run_rmsnorm(dev, stream, world, peaks, l2):
    """Fused RMSNorm + quantiser (bitlinear_rmsnorm_quant_act) against the
    plain quantiser (bitlinear_quant_act), bf16 rows; algorithmic bytes =
    2MK read + MK codes + 8M (eta, xsum) written."""
    from ternary_weight_linear_04_b200 import _lib, inputs
    L = _lib.lib()
    P = ctypes.c_void_p
    sptr = ctypes.c_void_p(stream.cuda_stream)
    hbm = float(peaks["hbm_gbs"])
    rng = np.random.default_rng(9)
    rows = []
    for M, K in ((1, 3200), (1, 8640), (64, 3200), (2048, 3200), (2048, 8640)):
        copies = max(1, min(64, int(np.ceil(3 * l2 / (2 * M * K)))))
        x0 = torch.from_numpy(inputs.draw_activations(rng, M, K, "normal", "bf16"))
        bufs = []
        for _ in range(copies):
            bufs.append(dict(x=x0.to(dev).to(torch.bfloat16),
                             xq=torch.empty((M, K), dtype=torch.int8, device=dev),
                             eta=torch.empty(M, dtype=torch.float32, device=dev),
                             xsum=torch.empty(M, dtype=torch.int32, device=dev)))
        torch.cuda.synchronize()
        res = {"M": M, "K": K, "copies": copies}
        nbytes = 3 * M * K + 8 * M
        for name, fn in (("rmsnorm_quant", L.bitlinear_rmsnorm_quant_act),
                         ("quant_only", L.bitlinear_quant_act)):
            calls = [lambda b=b, fn=fn: _chk(fn(P(b["x"].data_ptr()), _lib.BL_BF16, M, K,
                                               P(b["xq"].data_ptr()), P(b["eta"].data_ptr()),
                                               P(b["xsum"].data_ptr()), sptr), name)
                     for b in bufs]
            with torch.cuda.stream(stream):
                for c in calls:
                    c()
            torch.cuda.synchronize()
            gr = Capture(calls, stream)
            with torch.cuda.stream(stream):
                gr.replay()
            torch.cuda.synchronize()
            reps = max(3, 200 // copies)
            t = max_over_ranks(timed(lambda: [gr.replay() for _ in range(reps)], stream, world),
                               world) / (reps * copies)
            res[name] = {"us": round(t * 1e6, 2), "gbs": round(nbytes / t / 1e9, 1),
                         "hbm_frac": round(nbytes / t / 1e9 / hbm, 4)}
        rows.append(res)
        del bufs
        torch.cuda.empty_cache()
    return {"what": "RMSNorm (exact sum of squares) fused with the quantiser vs. the quantiser "
                    "alone; inputs rotate over copies (> 3x L2 where the rows allow, else "
                    "L2-resident, as in decode)", "rows": rows}


def run_pack(mats, stream, world):
    from ternary_weight_linear_04_b200 import bitlinear as bl
    m = mats[0]
    W = m["W"]
    N, K = W.shape
    from ternary_weight_linear_04_b200 import _lib
    ws = torch.empty(int(_lib.lib().bitlinear_pack_workspace_bytes()), dtype=torch.uint8, device=W.device)
    pk = torch.empty_like(m["packed"])
    g = torch.empty_like(m["gamma"])
    with torch.cuda.stream(stream):
        for _ in range(3):
            bl.pack_weights(W, stream=stream, workspace=ws, packed=pk, gamma=g)
    torch.cuda.synchronize()
    reps = 20
    with torch.cuda.stream(stream):
        t = timed(lambda: [bl.pack_weights(W, stream=stream, workspace=ws, packed=pk, gamma=g)
                           for _ in range(reps)], stream, world)
    t = max_over_ranks(t, world) / reps
    b = 2 * 4 * N * K + N * ((K + 3) // 4)
    return {"matrix": "%dx%d fp32" % (N, K), "us": round(t * 1e6, 1),
            "gbs": round(b / t / 1e9, 1),
            "note": "load-time: gamma from an fp64 sum of |W| under a proved bound (exact buckets only "
                    "when it cannot decide), then ternarise/pack by threshold (reads W twice)"}


def run_cpu_baseline(seconds):
    """The CPU oracle (scalar C, OpenMP over output rows) on the same
    workload, as it stands: about `seconds` seconds on every host thread,
    then about a third of that on one thread."""
    from oracle import native as orc
    from ternary_weight_linear_04_b200 import inputs
    wl = inputs.WORKLOADS[WORKLOAD]
    mats = []
    for j in range(len(wl.matrices)):
        W, x = inputs.make_matrix_inputs(wl, j, m_max=1)
        packed, gamma, _ = orc.pack_weights(W)
        mats.append((W.shape[1], W.shape[0], x, packed, gamma))
    b = sum(linear_bytes(1, K, N) for K, N, *_ in mats)

    def timed_steps(budget, nthreads):
        steps = 0
        t0 = time.perf_counter()
        while True:
            for K, N, x, packed, gamma in mats:
                xq, eta, _ = orc.quant_act(x)
                orc.forward(xq, eta, packed, gamma, K, N, nthreads=nthreads, want_y_int=False)
            steps += 1
            if time.perf_counter() - t0 >= budget:
                return steps, time.perf_counter() - t0

    threads = orc.max_threads()
    steps, t = timed_steps(seconds, 0)
    steps1, t1 = timed_steps(seconds / 3.0, 1)
    return {"value": round(b * steps / t / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": "%d full decode_3b steps (M=1, both matrices) in %.1f s on %d host threads"
                      % (steps, t, threads),
            "single_thread": {"value": round(b * steps1 / t1 / 1e9, 4), "unit": "GB/s",
                              "sample": "%d steps in %.1f s on 1 thread" % (steps1, t1)}}


# ----------------------------------------------------------------- profiling program

def profile_kernels():
    """Each kernel of the library, twice, at the size of the workload it
    serves (for ncu: capture the second launch of a kernel with -s 1 -c 1,
    or all of them): pack (decode_3b's 8640 x 3200 fp32 W), quantiser
    (prefill_7b's 2048 x 4096), RMSNorm + quantiser (2048 x 8640), the
    one-token decode kernel on both decode_3b matrices, the quantiser with
    the register-resident kernel for four tokens and with the warp-MMA
    kernel for sixteen (decode_3b K=3200 -> N=8640), the tensor-core kernel
    on prefill_7b, the base-3
    kernel on decode_3b (K=3200 -> N=8640) and the generic kernel (M = 3,
    K = 1000, N = 300)."""
    from ternary_weight_linear_04_b200 import build as libbuild, inputs
    from ternary_weight_linear_04_b200 import bitlinear as bl
    libbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = inputs.WORKLOADS["decode_3b"]
    mats = []
    for j in range(2):
        W, x = inputs.make_matrix_inputs(wl, j, m_max=16)
        mats.append((torch.from_numpy(W).to(dev), torch.from_numpy(x).to(dev).to(torch.bfloat16)))
    pw = inputs.WORKLOADS["prefill_7b"]
    Wp, xp = inputs.make_matrix_inputs(pw, 0)
    Wp = torch.from_numpy(Wp).to(dev)
    xp = torch.from_numpy(xp).to(dev).to(torch.bfloat16)
    rng = np.random.default_rng(5)
    xr = torch.from_numpy(inputs.draw_activations(rng, 2048, 8640, "normal", "bf16")).to(dev).to(torch.bfloat16)
    torch.cuda.synchronize()
    for _ in range(2):
        packed = [bl.pack_weights(W) for W, _ in mats]
        bl.quant_act(xp)
        bl.rmsnorm_quant_act(xr)
        for (pk, g), (W, x) in zip(packed, mats):
            bl.linear(x[:1], pk, g, W.shape[0], weights_static=True)
        pk, g = packed[0]
        bl.linear(mats[0][1][:4], pk, g, mats[0][0].shape[0], weights_static=True)
        bl.linear(mats[0][1][:16], pk, g, mats[0][0].shape[0], weights_static=True)
        ppk, pg = bl.pack_weights(Wp)
        xq, eta, xsum = bl.quant_act(xp)
        bl.forward(xq, eta, xsum, ppk, pg, Wp.shape[0], weights_static=True)
        p3, g3 = bl.pack_weights3(mats[0][0])
        xq1, eta1, xsum1 = bl.quant_act(mats[0][1][:1])
        bl.forward3(xq1, eta1, xsum1, p3, g3, mats[0][0].shape[0])
        Wg, xg = inputs.make_case(77, 3, 1000, 300)
        pkg, gg = bl.pack_weights(torch.from_numpy(Wg).to(dev))
        xqg, etag, xsg = bl.quant_act(torch.from_numpy(xg).to(dev))
        bl.forward(xqg, etag, xsg, pkg, gg, 300, path="generic")
        torch.cuda.synchronize()
    print(json.dumps({"profile_kernels": "done", "device": torch.cuda.get_device_name(dev)}))


# ----------------------------------------------------------------- reference arm

def run_reference(args, world, rank):
    """The CPU oracle timed on this machine's host cores: each step a bounded
    sample of the decode workload (a slice of output rows of both
    matrices), sized so warm-up + steps take about --ref-seconds (two
    minutes by default)."""
    if rank != 0:
        return None
    from oracle import native as orc
    from ternary_weight_linear_04_b200 import inputs
    wl = inputs.WORKLOADS[WORKLOAD]
    mats = []
    for j in range(len(wl.matrices)):
        W, x = inputs.make_matrix_inputs(wl, j, m_max=args.m)
        packed, gamma, _ = orc.pack_weights(W)
        mats.append((W.shape[1], W.shape[0], x, packed, gamma))
    threads = orc.max_threads()

    def step(frac):
        tot = 0
        for K, N, x, packed, gamma in mats:
            n = max(1, int(N * frac))
            xq, eta, _ = orc.quant_act(x)
            orc.forward(xq, eta, packed[:n], gamma, K, n, want_y_int=False)
            tot += linear_bytes(x.shape[0], K, n)
        return tot

    t0 = time.perf_counter()
    step(1.0)
    t_full = time.perf_counter() - t0
    budget = float(args.ref_seconds) / max(1, args.steps + args.warmup)
    frac = min(1.0, budget / max(t_full, 1e-9))
    for _ in range(args.warmup):
        step(frac)
    b = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        b += step(frac)
    t = time.perf_counter() - t0
    value = b / t / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": "decode_3b: K=3200->N=8640 and K=8640->N=3200, M=%d, bf16 in/out"
                                   % args.m, "M": args.m},
            "cpu_baseline": {"kind": "oracle", "cores": threads, "value": round(value, 4),
                             "unit": "GB/s",
                             "sample": "each step: %.4f of the output rows of both matrices" % frac},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--m", type=int, default=1, help="tokens per step (decode batch)")
    ap.add_argument("--quick", action="store_true", help="headline only (no e2e/prefill/pack)")
    ap.add_argument("--sections", default="",
                    help="comma list of extra sections: e2e,prefill,pack,sweep,layer70b,crossover,base3,"
                         "rmsnorm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-dir", default=None,
                    help="folder for the raw nvidia-smi clock samples (default: the temp folder)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="--impl reference: total CPU time of warm-up + timed steps")
    ap.add_argument("--windows", type=int, default=0,
                    help="number of timed windows of --steps steps (default: >= 5 and >= 50 ms)")
    ap.add_argument("--profile-kernels", action="store_true",
                    help="run each library kernel twice at its workload's size and exit "
                         "(a short program for ncu captures; prints one line)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args.gpus)
    if args.profile_kernels:
        profile_kernels()
        return
    try:
        if args.impl == "reference":
            out = run_reference(args, world, rank)
        else:
            out = run_ours(args, world, rank, local)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
