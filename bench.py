"""Benchmark of the Qwen-Image-2.1 joint-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
position table -> full block-causal step (axial RoPE, tile-skipping mask,
Prefix KV cache store) -> one prefix-cached target-only step.  The metric is
algorithmic TFLOP/s: 4 * 128 * (allowed query/key pairs) per (batch, head),
masked tiles and elements excluded.  For the max-reference workload the line
also carries ``loop``: the 8-step denoising loop of one layer (1 full + 7
cached steps on fresh target inputs) timed as eager calls and as one CUDA
graph replay.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload t2i]
    python bench.py --impl reference ...   # the float64 CPU oracle, timed

Multi-GPU (torchrun, one rank per GPU): every rank runs its own copy of the
workload (independent requests; no data exchange), the device time is the max
over ranks and ``value`` is the work of all ranks over that time (weak scaling).
Prints one JSON line on rank 0.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from diffusion_transformer_joint_axial_b200 import workloads as W  # noqa: E402

METRIC = "joint-attn TFLOP/s (full step & prefix-cached step), % of B200 BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per attention call -- the rotation/cache
# pre-pass plus the attention kernel -- from one ncu capture of each kernel
# (dram__bytes_read.sum + dram__bytes_write.sum), per workload.  Valid only for
# the kernel sources they were taken on: any other source reports null.
NCU_TRAFFIC = {"sources_sha256": "d9e77a0f51985532",
               # mean of the full and the cached call
               "bytes_per_call": {"t2i": ((28.399e6 + 0.098e6 + 82.082e6 + 2.291e6)
                                          + (25.250e6 + 0.000e6 + 79.879e6 + 1.046e6)) / 2,
                                  "hires": ((315.112e6 + 262.514e6 + 2569.402e6 + 276.766e6)
                                            + (201.684e6 + 144.807e6 + 2396.354e6 + 231.838e6)) / 2}}


def kernel_sources_digest(read=None):
    """Hash of the attention and pre-pass kernels' code (and the device
    helpers they include) with // comments and blank lines dropped, so that
    editing a comment keeps the recorded traffic."""
    h = hashlib.sha256()
    for name in ("attn_tc.cu", "prep_kernels.cu", "qi21_device.cuh"):
        if read is None:
            with open(os.path.join(ROOT, "diffusion_transformer_joint_axial_b200", "csrc", name)) as f:
                text = f.read()
        else:
            text = read(name)
        for line in text.splitlines():
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def ncu_traffic(name):
    if NCU_TRAFFIC["sources_sha256"] != kernel_sources_digest():
        return None
    return NCU_TRAFFIC["bytes_per_call"].get(name)


# ------------------------------------------------------------------ helpers --

def step_flops(name):
    """Algorithmic FLOPs of one step: full step + one cached step, all heads
    (the earlier model's workload: one unmasked full step, no cached step)."""
    cfg = W.WORKLOADS[name]
    L, P, T = W.sizes(name)
    if cfg.get("original"):
        return 4.0 * 128 * L * L * cfg["B"] * cfg["H"], 0.0
    # allowed pairs of the full step: sum over rows of their visibility bound
    # (the segment layout fixes it: text token i sees i + 1 keys, an image
    # token sees everything up to the end of its image)
    pairs = 0
    start = 0
    for s in cfg["segments"]:
        n = W.seg_tokens(s)
        if s["kind"] == "text":
            pairs += n * start + n * (n + 1) // 2
        else:
            pairs += n * (start + n)
        start += n
    full = 4.0 * 128 * pairs * cfg["B"] * cfg["H"]
    cached = 4.0 * 128 * T * (P + T) * cfg["B"] * cfg["H"]
    return full, cached


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons sampled on a background thread (NVML)
    while the timed regions run; falls back to ``nvidia-smi -lms`` polling.
    Only samples taken between ``start()`` and ``pause()`` count, so several
    short timed regions add up to one record."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device):
        import threading
        self.sm, self.reasons, self.power = [], set(), []
        self.sm_max = None
        self.active = threading.Event()
        self.done = threading.Event()
        self.handle = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device)
            bus = "%08X:%02X:%02X.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                         props.pci_device_id)
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except pynvml.NVMLError:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.nvml = pynvml
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: nothing recorded, and the record says why
            self.error = "NVML unavailable (%s)" % type(e).__name__
            return
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def _loop(self):
        nv = self.nvml
        while not self.done.is_set():
            if self.active.wait(0.05):
                try:
                    self.sm.append(float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)))
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    for name, bit in self.REASONS:
                        if r & bit:
                            self.reasons.add(name)
                    self.power.append(nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0)
                except Exception:
                    pass
                time.sleep(0.002)

    def start(self):
        self.active.set()

    def pause(self):
        self.active.clear()

    def stop(self):
        self.pause()
        self.done.set()
        if self.error:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error], "samples": 0}
        self.thread.join(timeout=5)
        return {"sm_mhz": statistics.median(self.sm) if self.sm else None, "sm_max_mhz": self.sm_max,
                "reasons": sorted(self.reasons), "samples": len(self.sm),
                "power_w_max": max(self.power) if self.power else None, "source": "NVML, 2 ms polling"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            backend="nccl" if torch.cuda.is_available() else "gloo",
            timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x, world, device):
    """Max of a per-rank float over all ranks (identity on one rank)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device):
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ---------------------------------------------------------------- CPU oracle --

ORACLE_ROWS = 512  # query rows per oracle piece


def oracle_sample(name, budget_s, max_pieces=None):
    """Times the float64 oracle on a bounded sample of the workload: pieces of
    ORACLE_ROWS query rows of one head, one piece of the full step (rows taken
    in turn along the sequence, so text, reference and target rows all come
    up) plus one piece of the cached step, until ``budget_s`` passes (at least
    one piece).  Returns (algorithmic flops of the rows done, seconds, pieces)."""
    import oracle as O
    cfg = W.WORKLOADS[name]
    L, P, T = W.sizes(name)
    q, k, v = W.draw_qkv(1, L, 1, cfg["seed"], cfg["dtype"])
    qf, kf, vf = W.as_f64(q), W.as_f64(k), W.as_f64(v)
    orig = cfg.get("original", False)
    pos, kv_end = (O.positions_original if orig else O.positions)(cfg["segments"])
    kv_end = np.asarray(kv_end, dtype=np.int64)
    kc = vc = None
    flops, pieces = 0.0, 0
    t0 = time.perf_counter()
    while True:
        r0 = (pieces * ORACLE_ROWS) % L
        rows = np.arange(r0, min(L, r0 + ORACLE_ROWS))
        O.attn_full(qf, kf, vf, pos, kv_end, rows=rows)
        flops += 4.0 * 128 * float(kv_end[rows].sum())
        if not orig:
            if kc is None:
                kc, vc = O.prefix_cache(kf, vf, pos, P)
            c0 = (pieces * ORACLE_ROWS) % T
            crows = np.arange(c0, min(T, c0 + ORACLE_ROWS))
            O.attn_cached(qf[:, P:], kf[:, P:], vf[:, P:], pos[P:], kc, vc, rows=crows)
            flops += 4.0 * 128 * len(crows) * (P + T)
        pieces += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s or (max_pieces is not None and pieces >= max_pieces):
            return flops, dt, pieces


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, world, rank):
    """The reference arm: the float64 oracle (the only CPU implementation of
    the method) timed on the host cores, one oracle piece per step, on the
    headline workload's shapes; rank 0 only."""
    if rank != 0:
        return
    name = headline_workload(args)
    cfg = W.WORKLOADS[name]
    for _ in range(args.warmup):
        oracle_sample(name, 0.0, max_pieces=1)
    tot_f, tot_s, pieces = 0.0, 0.0, 0
    for _ in range(args.steps):
        f, s, n = oracle_sample(name, 0.0, max_pieces=1)
        tot_f, tot_s, pieces = tot_f + f, tot_s + s, pieces + n
    value = tot_f / tot_s / 1e12
    sample = ("per step: %d query rows of one head of the %s full step%s (float64 NumPy oracle); "
              "TFLOP/s counts the algorithmic work of the rows done" % (
                  ORACLE_ROWS, name, "" if cfg.get("original") else " + %d rows of its cached step" % ORACLE_ROWS))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_s / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": W.DESCRIPTIONS[name], "B": cfg["B"], "H": cfg["H"]},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm --

def pct(xs, q):
    return float(np.percentile(np.asarray(xs, dtype=np.float64), q))


def time_projections(qi, args, M, D, flush, dev):
    """tcgen05 projections of the target tokens of a cached step: the fused
    Q/K/V projection (N = 3 D, three outputs) and the output projection
    (N = D), bf16 with synthetic seeded weights; cuBLAS (torch.matmul) on the
    same shapes for context.  L2 flushed before each rep."""
    g = torch.Generator(device="cpu").manual_seed(11)
    mk = lambda *shape, scale=1.0: (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16).to(dev)
    x = mk(M, D)
    w_qkv, b_qkv = mk(3 * D, D, scale=D ** -0.5), mk(3 * D, scale=0.1)
    w_o, b_o = mk(D, D, scale=D ** -0.5), mk(D, scale=0.1)
    ws = qi.new_workspace(256, dev)
    outs = [torch.empty((M, D), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    y = torch.empty((M, D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    reps = max(3, min(args.steps, 20))
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(fn):
        for _ in range(3):
            fn()
        pairs = [(ev(), ev()) for _ in range(reps)]
        for a, b in pairs:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return pct([a.elapsed_time(b) for a, b in pairs], 50)

    out = {"M": M, "hidden": D, "weights": "synthetic N(0, 1/hidden), bias N(0, 0.01)", "reps": reps}
    for name, w, b, o, n_out in (("qkv", w_qkv, b_qkv, outs, 3), ("out", w_o, b_o, [y], 1)):
        flops = 2.0 * M * w.shape[0] * D
        ms = timed(lambda: qi.linear(x, w, b, n_out=n_out, out=o, workspace=ws))
        ms_ref = timed(lambda: torch.addmm(b, x, w.t()))
        out[name] = {"N": int(w.shape[0]), "ms": ms, "tflops": flops / (ms * 1e-3) / 1e12,
                     "cublas_tflops": flops / (ms_ref * 1e-3) / 1e12}
    assert qi.workspace_status(ws) == 0
    return out


def time_denoise(qi, args, cfg, dev):
    """The denoising loop around the attention on this workload's layout:
    ``--denoise-blocks`` blocks (attention + SwiGLU), 8 Euler steps, random
    weights drawn on the device (N(0, 1/fan_in); biases 0.02 N(0, 1)), 64
    latent channels.  One graph replay = one whole loop (step 1 on every
    token, steps 2..8 on the target tokens against the per-block caches).
    Also runs the full recomputation once from the same latents and reports
    the largest difference (the cache-reuse check)."""
    steps, C, nb, H = 8, 64, args.denoise_blocks, cfg["H"]
    sig = W.denoise_sigmas(steps)
    gen = torch.Generator(device=dev)
    gen.manual_seed(13)
    D, F = H * 128, 3 * H * 128
    rnd = lambda *shape, scale=1.0, shift=0.0: (torch.randn(*shape, generator=gen, device=dev) * scale
                                                 + shift).to(torch.bfloat16)
    blk = lambda: dict(norm1=rnd(D, scale=0.1, shift=1.0), w_qkv=rnd(3 * D, D, scale=D ** -0.5),
                       b_qkv=rnd(3 * D, scale=0.02), w_o=rnd(D, D, scale=D ** -0.5), b_o=rnd(D, scale=0.02),
                       norm2=rnd(D, scale=0.1, shift=1.0), w_gu=rnd(2 * F, D, scale=D ** -0.5),
                       b_gu=rnd(2 * F, scale=0.02), w_down=rnd(D, F, scale=F ** -0.5), b_down=rnd(D, scale=0.02))
    params = dict(w_in=rnd(D, C, scale=C ** -0.5), b_in=rnd(steps, D, scale=0.5), blocks=[blk() for _ in range(nb)],
                  norm_out=rnd(D, scale=0.1, shift=1.0), w_v=rnd(C, D, scale=D ** -0.5), b_v=rnd(C, scale=0.02))
    segs = cfg["segments"]
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    x0, ph = rnd(1, T, C), rnd(1, L - T, D)
    model = qi.denoise.DenoiseModel(segs, H, C, nb, steps, sig, device=dev, cached=True)
    model.load(params, x0, ph)
    model.run()
    model.check()
    x_cached = model.x.clone()
    model.x.copy_(x0)
    model.capture()
    reps = max(2, min(args.steps, 5))
    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps + 1)]
    for i, (a, b) in enumerate(ev):  # the first replay is a warm-up
        a.record(stream)
        model.replay()
        b.record(stream)
    torch.cuda.synchronize()
    model.check()
    ms = pct([a.elapsed_time(b) for a, b in ev[1:]], 50)
    flops = model.flops()
    del model
    torch.cuda.empty_cache()
    full = qi.denoise.DenoiseModel(segs, H, C, nb, steps, sig, device=dev, cached=False)
    full.load(params, x0, ph)
    full.run()
    full.check()
    diff = (full.x.float() - x_cached.float()).abs()
    out = {"blocks": nb, "steps": steps, "heads": H, "channels": C, "tokens": L, "target_tokens": T,
           "graph_ms_median": ms, "tflop_per_loop": flops / 1e12, "tflops": flops / (ms * 1e-3) / 1e12,
           "cached_vs_full_max_abs": float(diff.max()), "cached_vs_full_mean_abs": float(diff.mean()),
           "latent_rms": float(x_cached.float().pow(2).mean().sqrt()),
           "what": "reduced loop: embedding, blocks of RMSNorm/attention/SwiGLU with residuals, velocity, "
                   "Euler; random weights on the device"}
    del full
    torch.cuda.empty_cache()
    return out


def time_loop(qi, args, name, cfg, flush, dev, full_flops, cached_flops):
    """The workload's denoising loop for one layer: step 1 full (cache store)
    and steps 2..N cached on fresh target inputs, timed eagerly (one library
    call per step) and as one CUDA-graph replay; L2 flushed before each."""
    n = 1 + cfg["cached_steps"]
    loop = qi.DenoiseLoop(cfg["segments"], cfg["B"], cfg["H"], n, torch.bfloat16, dev)
    loop.load(*W.full_inputs(name), [W.cached_inputs(name, s) for s in range(2, n + 1)])
    loop.capture()
    stream = torch.cuda.current_stream(dev)
    reps = max(3, min(args.steps, 10))
    mk = lambda: torch.cuda.Event(enable_timing=True)
    times = {}
    for mode, fn in (("eager", loop.run), ("graph", loop.replay)):
        for _ in range(2):
            fn()
        ev = [(mk(), mk()) for _ in range(reps)]
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        times[mode] = [a.elapsed_time(b) for a, b in ev]
    loop.check()
    flops = full_flops + (n - 1) * cached_flops
    g = pct(times["graph"], 50)
    out = {"steps": n, "calls": "1 full + %d cached" % (n - 1), "reps": reps,
           "graph_ms_median": g, "graph_ms_p95": pct(times["graph"], 95),
           "eager_ms_median": pct(times["eager"], 50), "eager_ms_p95": pct(times["eager"], 95),
           "tflops_graph": flops / (g * 1e-3) / 1e12}
    del loop
    torch.cuda.empty_cache()

    # the same loop as attention sublayers: projections of each step's tokens
    # (step 1 all L, later steps the T target tokens) around the attention
    B, H = cfg["B"], cfg["H"]
    L, P, T = W.sizes(name)
    D = H * 128
    layer = qi.DenoiseLoop(cfg["segments"], B, H, n, torch.bfloat16, dev, projections=True)
    g = torch.Generator(device="cpu").manual_seed(12)
    rnd = lambda *shape, scale=1.0: (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)
    layer.load_layer(rnd(B, L, D), [rnd(B, T, D) for _ in range(n - 1)], rnd(3 * D, D, scale=D ** -0.5),
                     rnd(3 * D, scale=0.1), rnd(D, D, scale=D ** -0.5), rnd(D, scale=0.1))
    layer.capture()
    for _ in range(2):
        layer.replay()
    ev = [(mk(), mk()) for _ in range(reps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        layer.replay()
        b.record(stream)
    torch.cuda.synchronize()
    layer.check()
    lt = [a.elapsed_time(b) for a, b in ev]
    proj_flops = 2.0 * 4 * D * D * B * (L + (n - 1) * T)  # Q/K/V (3 D x D) + output (D x D)
    gl = pct(lt, 50)
    out["layer"] = {"what": "attention sublayer: fused Q/K/V projection -> attention -> output projection, "
                            "synthetic weights; step 1 projects all %d tokens, steps 2..%d the %d target "
                            "tokens" % (L, n, T),
                    "graph_ms_median": gl, "graph_ms_p95": pct(lt, 95),
                    "tflops_graph": (flops + proj_flops) / (gl * 1e-3) / 1e12,
                    "projection_tflop": proj_flops / 1e12}
    del layer
    torch.cuda.empty_cache()
    return out


BENCH_WORKLOADS = ("t2i", "edit3", "maxref", "hires", "orig")
# The largest single-GPU configuration (B=2, 16384 target tokens): the line's headline.
HEADLINE = "hires"


def headline_workload(args):
    return HEADLINE if args.workload == "all" else args.workload


def bench_workload(qi, args, name, world, dev, flush, clocks, headline):
    """Times ``args.steps`` steps of one workload after ``args.warmup``
    untimed ones.  A step = positions -> full block-causal step with cache
    store -> one cached step (the earlier model's layout: positions -> one
    unmasked full step), each a whole C-ABI call (its rotation/cache pre-pass
    and its attention kernel) bracketed by CUDA events on the launch stream;
    L2 is flushed before every step, outside the events.  Returns the record
    of the workload (times are max over ranks) and, for the headline, the raw
    numbers the JSON line is made of."""
    lib = qi.load_library()
    cfg = W.WORKLOADS[name]
    B, H = cfg["B"], cfg["H"]
    L, P, T = W.sizes(name)
    segs = cfg["segments"]
    dt = torch.bfloat16
    orig = cfg.get("original", False)
    q, k, v = W.full_inputs(name)
    host = [x.pin_memory() for x in ((q, k, v) if orig else (q, k, v) + tuple(W.cached_inputs(name, 2)))]
    dq, dk, dv = (x.to(dev) for x in host[:3])
    dqt, dkt, dvt = (None, None, None) if orig else (x.to(dev) for x in host[3:])
    kc, vc = (None, None) if orig else qi.alloc_cache(B, H, P, dt, dev)
    o_full = torch.empty_like(dq)
    o_c = None if orig else torch.empty_like(dqt)
    ws_f = qi.new_workspace(qi.full_workspace_size(B, H, L, 0 if orig else P, dt), dev)
    ws_c = qi.new_workspace(256 if orig else qi.cached_workspace_size(B, H, P, T, dt), dev)
    pos = torch.empty((L, 3), dtype=torch.int32, device=dev)
    kv_end = torch.empty((L,), dtype=torch.int32, device=dev)
    assert pos[P:].data_ptr() % 16 == 0, "target rows of the position table must be 16-byte aligned"
    seg_arr = qi._binding.to_segments(segs)
    stream = torch.cuda.current_stream(dev)
    sp = qi._binding.ctypes.c_void_p(stream.cuda_stream)
    P_ = qi._binding._ptr
    if args.qk_norm:  # the fused QK-RMSNorm variant of both steps
        wq, wk = (w.to(dev) for w in W.qk_norm_weights())
        norm = (P_(wq), P_(wk), qi._binding.ctypes.c_float(W.QK_NORM_EPS))
        full_fn = lambda *a: lib.qi21_attn_full_qknorm(*a[:13], *norm, *a[13:])
        cached_fn = lambda *a: lib.qi21_attn_cached_qknorm(*a[:12], *norm, *a[12:])
    else:
        full_fn, cached_fn = lib.qi21_attn_full, lib.qi21_attn_cached
    positions_fn = lib.qi21_rope_positions_original if orig else lib.qi21_rope_positions
    # the earlier model attends without a mask: kv_end NULL (every key visible)
    kv_arg = None if orig else kv_end

    def one_step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        st = positions_fn(seg_arr, len(segs), L, P_(pos), P_(kv_end), sp)
        assert st == 0, lib.qi21_last_error()
        if ev is not None:
            ev[1].record(stream)
        st = full_fn(B, H, L, 0 if orig else P, 0, P_(dq), P_(dk), P_(dv), P_(pos), P_(kv_arg), P_(o_full),
                     P_(kc), P_(vc), P_(ws_f), ws_f.numel(), sp)
        assert st == 0, lib.qi21_last_error()
        if ev is not None:
            ev[2].record(stream)
        if not orig:
            st = cached_fn(B, H, P, T, 0, P_(dqt), P_(dkt), P_(dvt), P_(pos[P:]), P_(kc), P_(vc),
                           P_(o_c), P_(ws_c), ws_c.numel(), sp)
            assert st == 0, lib.qi21_last_error()
        if ev is not None:
            ev[3].record(stream)

    full_flops, cached_flops = step_flops(name)
    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    assert qi.workspace_status(ws_f) == 0 and qi.workspace_status(ws_c) == 0

    mk = lambda: torch.cuda.Event(enable_timing=True)
    evs = [(mk(), mk(), mk(), mk()) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    n0 = qi.launch_count()
    for e in evs:
        flush.zero_()
        one_step(e)
    torch.cuda.synchronize()
    if clocks:
        clocks.pause()
    barrier(world)
    launches = qi.launch_count() - n0
    assert qi.workspace_status(ws_f) == 0 and qi.workspace_status(ws_c) == 0
    step_each = [e[0].elapsed_time(e[3]) for e in evs]
    pos_each = [e[0].elapsed_time(e[1]) for e in evs]
    full_each = [e[1].elapsed_time(e[2]) for e in evs]
    cached_each = [e[2].elapsed_time(e[3]) for e in evs]
    K = args.steps
    step_ms = max_over_ranks(sum(step_each), world, dev)
    full_ms = max_over_ranks(sum(full_each), world, dev)
    cached_ms = max_over_ranks(sum(cached_each), world, dev)
    peak = load_peaks()[0]["bf16_tflops"]

    def step_record(flops, ms_total, each):
        tf = world * flops * K / (ms_total * 1e-3) / 1e12
        return {"tflop": flops / 1e12, "ms": ms_total / K, "ms_median": pct(each, 50), "ms_p95": pct(each, 95),
                "tflops": tf, "frac_of_peak": tf / peak / world}

    rec = {"workload": W.DESCRIPTIONS[name], "B": B, "H": H, "L": L, "P": P, "T": T,
           "full_step": step_record(full_flops, full_ms, full_each),
           "cached_step": None if orig else step_record(cached_flops, cached_ms, cached_each),
           "positions_ms_median": pct(pos_each, 50),
           "step": {"ms": step_ms / K, "tflops": world * (full_flops + cached_flops) * K / (step_ms * 1e-3) / 1e12},
           "gpu_launches": launches}
    # per-rank throughput used for the line's aggregate value
    raw = {"flops_per_step": full_flops + cached_flops, "step_ms": step_ms, "full_ms": full_ms,
           "cached_ms": cached_ms, "launches": launches}

    if name == "maxref" and not args.qk_norm:
        rec["loop"] = time_loop(qi, args, name, cfg, flush, dev, full_flops, cached_flops)

    if headline:
        # End to end through the C ABI with host buffers: every step copies its
        # inputs from pinned host memory and reads its outputs back, as a
        # serving loop would run it -- copies in, compute and copies out on
        # three streams with double-buffered device tensors, so that a step's
        # cached-call inputs go up while its full call runs and its outputs
        # come down while the next step computes.  One timed region from the
        # first copy in to the last copy out.
        h2d = sum(x.numel() * x.element_size() for x in host)
        outs_d = [o_full] if orig else [o_full, o_c]
        d2h = sum(o.numel() for o in outs_d) * 2
        out_h = [torch.empty(o.shape, dtype=dt, pin_memory=True) for o in outs_d]
        e2e_steps = max(3, min(K, 20))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ins = [[dq, dk, dv] + ([] if orig else [dqt, dkt, dvt])]
        ins.append([torch.empty_like(x) for x in ins[0]])
        outs = [outs_d, [torch.empty_like(o) for o in outs_d]]
        ev = lambda: torch.cuda.Event()
        in_free = [None, None]   # compute done with a slot's inputs
        out_free = [None, None]  # copies out done with a slot's outputs
        t_start, t_end = mk(), mk()
        barrier(world)
        torch.cuda.synchronize()
        t_start.record(s_in)
        for i in range(e2e_steps):
            sl = i % 2
            d_in, d_out = ins[sl], outs[sl]
            full_in, cached_in = ev(), ev()
            with torch.cuda.stream(s_in):
                if in_free[sl] is not None:
                    s_in.wait_event(in_free[sl])
                for d, h in zip(d_in[:3], host[:3]):
                    d.copy_(h, non_blocking=True)
                full_in.record(s_in)
                for d, h in zip(d_in[3:], host[3:]):
                    d.copy_(h, non_blocking=True)
                cached_in.record(s_in)
            stream.wait_event(full_in)
            if out_free[sl] is not None:
                stream.wait_event(out_free[sl])
            flush.zero_()
            spn = qi._binding.ctypes.c_void_p(stream.cuda_stream)
            st = positions_fn(seg_arr, len(segs), L, P_(pos), P_(kv_end), spn)
            assert st == 0, lib.qi21_last_error()
            st = full_fn(B, H, L, 0 if orig else P, 0, P_(d_in[0]), P_(d_in[1]), P_(d_in[2]), P_(pos), P_(kv_arg),
                         P_(d_out[0]), P_(kc), P_(vc), P_(ws_f), ws_f.numel(), spn)
            assert st == 0, lib.qi21_last_error()
            full_done = ev()
            full_done.record(stream)
            if not orig:
                stream.wait_event(cached_in)
                st = cached_fn(B, H, P, T, 0, P_(d_in[3]), P_(d_in[4]), P_(d_in[5]), P_(pos[P:]), P_(kc), P_(vc),
                               P_(d_out[1]), P_(ws_c), ws_c.numel(), spn)
                assert st == 0, lib.qi21_last_error()
            step_done = ev()
            step_done.record(stream)
            in_free[sl] = step_done
            with torch.cuda.stream(s_out):
                s_out.wait_event(full_done)
                out_h[0].copy_(d_out[0], non_blocking=True)
                if not orig:
                    s_out.wait_event(step_done)
                    out_h[1].copy_(d_out[1], non_blocking=True)
                done = ev()
                done.record(s_out)
                out_free[sl] = done
        t_end.record(s_out)
        torch.cuda.synchronize()
        assert qi.workspace_status(ws_f) == 0 and qi.workspace_status(ws_c) == 0
        e2e_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
        raw["e2e"] = {"value": world * (full_flops + cached_flops) * e2e_steps / (e2e_ms * 1e-3) / 1e12,
                      "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                      "pipeline": "copies in / compute / copies out on three streams, double-buffered"}
        if name == "t2i" or args.workload != "all":
            rec["projections"] = time_projections(qi, args, B * T, H * 128, flush, dev)
        if args.denoise and not orig:
            rec["denoise"] = time_denoise(qi, args, cfg, dev)
    elif name == "t2i":
        rec["projections"] = time_projections(qi, args, B * T, H * 128, flush, dev)
    del dq, dk, dv, dqt, dkt, dvt, kc, vc, o_full, o_c, ws_f, ws_c, host
    torch.cuda.empty_cache()
    return rec, raw


def run_ours(args, world, rank, local):
    import diffusion_transformer_joint_axial_b200 as qi
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    head = headline_workload(args)
    names = BENCH_WORKLOADS if args.workload == "all" else (args.workload,)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2
    clocks = ClockSampler(dev) if rank == 0 else None
    records, raw_head = {}, None
    try:
        for name in names:
            assert W.WORKLOADS[name]["dtype"] == "bf16", "the bench measures the bf16 workloads"
            rec, raw = bench_workload(qi, args, name, world, dev, flush, clocks, name == head)
            records[name] = rec
            if name == head:
                raw_head = raw
    finally:
        clk = clocks.stop() if clocks else None
    if rank != 0:
        return

    peaks, kind = load_peaks()
    peak = peaks["bf16_tflops"]
    cfg = W.WORKLOADS[head]
    L, P, T = W.sizes(head)
    orig = cfg.get("original", False)
    K = args.steps
    hr = records[head]
    value = hr["step"]["tflops"]
    call_ms = raw_head["full_ms"] + raw_head["cached_ms"]
    achieved = world * raw_head["flops_per_step"] * K / (call_ms * 1e-3) / 1e12 / world

    # the oracle baseline runs on rank 0 of a one-GPU run only
    budget = 0.0 if (args.no_cpu_baseline or world > 1) else args.cpu_budget
    cpu = None
    if budget > 0:
        f, s, pieces = oracle_sample(head, budget)
        cpu = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": "%d pieces of %d query rows of one head of the %s %s (float64 NumPy oracle, "
                         "%.1f s; the rows cycle along the sequence)" % (
                             pieces, ORACLE_ROWS, head,
                             "unmasked full step" if orig else "full step + its cached step", s)}
    power_note = None
    if clk and "sw_power_cap" in (clk.get("reasons") or []):
        power_note = ("sw_power_cap was active during the timed regions; the fractions still use the "
                      "burst peak")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": hr["step"]["ms"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": W.DESCRIPTIONS[head], "B": cfg["B"], "H": cfg["H"], "L": L, "P": P, "T": T,
                   "step": ("positions (text after the images) + one unmasked full step" if orig else
                            "positions + full block-causal step with cache store + one cached step")
                           + (", QK-RMSNorm fused (synthetic weights)" if args.qk_norm else ""),
                   "timing": "whole C-ABI calls (rotation/cache pre-pass + attention kernel), CUDA events "
                             "on the launch stream",
                   "qk_norm": bool(args.qk_norm),
                   "k_rotation": args.k_rotation,
                   "l2": "flushed between steps (256 MiB write, outside the timed events)",
                   "parallelism": "dp%d (independent requests per GPU)" % world},
        "full_step": hr["full_step"],
        "cached_step": hr["cached_step"],
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": ncu_traffic(head) if args.k_rotation == "pre-pass" else None,
                     "traffic_unit": "bytes/call",
                     "kernel": "attention calls of the step (full + cached): rotation/cache pre-pass + "
                               "qi21::tc::attn_tc_kernel",
                     "peak_kind": "%s bf16 dense burst (cuBLAS), MEASURED_PEAKS.json" % kind
                                  if kind == "measured" else "fallback bf16 dense burst (1.59 PFLOP/s)"},
        "cpu_baseline": cpu,
        "e2e": raw_head["e2e"],
        "gpu_launches": raw_head["launches"],
        "clocks": clk,
        "power_note": power_note,
        "workloads": records,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="all",
                    choices=["all"] + [n for n in W.WORKLOADS if n != "tiny"],
                    help="all (default): every bf16 workload, the 2048^2 one as the headline")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--denoise", action="store_true",
                    help="also time the whole denoising loop (blocks of attention + SwiGLU, 8 Euler steps)")
    ap.add_argument("--denoise-blocks", type=int, default=32)
    ap.add_argument("--qk-norm", action="store_true",
                    help="time the variant with the QK-RMSNorm fused in front of RoPE")
    ap.add_argument("--k-rotation", default="pre-pass", choices=["pre-pass", "attention"],
                    help="where the keys outside the Prefix cache are rotated: once per token in "
                         "the pre-pass (default), or per key tile inside the attention kernel "
                         "(an ablation, sets QI21_K_ROTATION)")
    args = ap.parse_args(argv)
    if args.k_rotation == "attention":
        os.environ["QI21_K_ROTATION"] = "attention"
    else:
        os.environ.pop("QI21_K_ROTATION", None)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
