"""Throughput of the quantized recurrent-state decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lrs|reference]
                    [--workload NAME] [--layers L] [--mode rtn|sr|bdr] [--no-extras]

A step is one decode step of one layer's state: every (batch, head) tile of
the workload is dequantized, updated, read out and requantized once (one
kernel launch). Steps rotate over L independent layer states whose total size
is far above the 126 MB L2, as in a model where the other layers run between
two steps of one layer, so every step reads its state from HBM.

Prints one JSON line (rank 0). Under torchrun each rank runs its own batch of
the workload (weak scaling, no collective on the data path); the time is the
slowest rank's.

--impl reference times the CPU oracle on the host cores on a bounded sample of
tiles per step and reports the same metric for the whole workload.
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-state decode steps/s and state GB/s (% of HBM peak), B=256 32h 128×128"
DEFAULT_WORKLOAD = "gla_rtn_int8_b256h32_128"
MODES = {"rtn": 0, "sr": 1, "bdr": 2}
KERNEL_SOURCES = ["quantized_recurrent_state_decode_b200/csrc/step_kernel.cuh",
                  "quantized_recurrent_state_decode_b200/csrc/step_instances.cuh",
                  "quantized_recurrent_state_decode_b200/csrc/lrs_device.cuh",
                  "quantized_recurrent_state_decode_b200/csrc/step_rtn.cu"]
PROFILE = os.path.join(ROOT, "profiles", "step_kernel_gla_rtn_int8_b256h32.md")


def kernel_source_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def profiled_traffic():
    """DRAM bytes per launch of the step kernel from the committed ncu summary,
    if it was taken on the current kernel source; else None."""
    try:
        text = open(PROFILE).read()
    except OSError:
        return None
    m = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    t = re.search(r"dram_bytes_per_launch_full_workload:\s*([0-9.eE+]+)", text)
    if not m or not t or m.group(1) != kernel_source_hash():
        return None
    return float(t.group(1))


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        return time.time()

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(2)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [l for (ts, l) in self.lines if t0 <= ts <= t1] or \
            [l for (_, l) in self.lines[-5:]]
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# --------------------------------------------------------------- reference ---

class OracleSampler:
    """The CPU oracle on the host cores over a fixed, seeded sample of tiles of
    the workload. A pool of one thread per core is created once; each step
    hands every thread one contiguous slice of the sample (the oracle's C code
    runs single-threaded per call, outside the interpreter lock). Both CPU
    legs of the benchmark -- `--impl reference` and the GPU arm's
    `cpu_baseline` -- time through this one sampler, so they report one
    number for one workload."""

    def __init__(self, w, mode, ntiles=None, seed=0):
        import concurrent.futures as cf
        import numpy as np
        import oracle
        from quantized_recurrent_state_decode_b200 import inputs as I
        self.w, self.mode = w, mode
        self.nthreads = oracle.default_threads()
        n_all = w.batch * w.heads
        n = ntiles if ntiles else max(self.nthreads * 16, 256)
        n = min(n_all, n)
        rng = np.random.default_rng(seed)
        tiles = np.sort(rng.choice(n_all, size=n, replace=False))
        self.tb = (tiles // w.heads).astype(np.int32)
        self.th = (tiles % w.heads).astype(np.int32)
        self.n, self.n_all = n, n_all
        self.pm = oracle_precision_map(w)
        S0 = I.initial_state(w)[self.tb, self.th].numpy()
        self.codes, self.scales = oracle.import_fp32(S0, self.pm, self.th, group=w.group)
        self.xs = []
        for t in range(4):
            x = I.step_inputs(w, t)
            self.xs.append({k: (None if v is None else v[self.tb, self.th].numpy().reshape(n, -1))
                            for k, v in x.items()})
        T = self.nthreads
        self.slices = [slice(n * i // T, n * (i + 1) // T) for i in range(T)]
        self.slices = [sl for sl in self.slices if sl.stop > sl.start]
        self.pool = cf.ThreadPoolExecutor(len(self.slices))

    def _part(self, sl, x, t):
        import numpy as np
        import oracle
        w = self.w
        codes, scales = self.codes[sl], self.scales[sl]      # contiguous views, updated in place
        sel = {k: (None if v is None else v[sl]) for k, v in x.items()}
        oracle.step(codes, scales, sel["q"], sel["k"], sel["v"], sel["gates"],
                    None if sel["beta"] is None else sel["beta"].reshape(-1), self.pm,
                    self.tb[sl], self.th[sl], group=w.group, update_kind=w.update_kind,
                    gate_kind=w.gate_kind, mode=self.mode, seed=1, step=t, nthreads=1)

    def step(self, t):
        """One step over the sample; returns its wall time in seconds."""
        x = self.xs[t % len(self.xs)]
        t0 = time.perf_counter()
        list(self.pool.map(lambda sl: self._part(sl, x, t), self.slices))
        return time.perf_counter() - t0

    def steps_per_s(self, sec_per_sample_step):
        """Whole-workload steps/s from the time of one step over the sample."""
        return 1.0 / (sec_per_sample_step / self.n * self.n_all)

    def describe(self, steps, el):
        return ("%d of %d tiles per step (seeded sample), %d steps, %.1f s of oracle time on "
                "%d threads created once, scaled to the whole workload"
                % (self.n, self.n_all, steps, el, len(self.slices)))

    def close(self):
        self.pool.shutdown()


def run_reference(args, w):
    """The CPU oracle on the host cores: W untimed and K timed steps, each one
    step over the seeded tile sample; the metric is scaled to the workload."""
    mode = MODES[args.mode] if args.mode else w.mode
    smp = OracleSampler(w, mode)
    # a bounded sample: at most ~150 s for the whole run
    t1 = smp.step(0)
    reps = max(1, min(16, int(150.0 / max(t1, 1e-3) / max(args.steps + args.warmup, 1))))
    for t in range(args.warmup):
        for _ in range(reps):
            smp.step(t)
    el = 0.0
    for t in range(args.steps):
        for _ in range(reps):
            el += smp.step(t)
    smp.close()
    steps_per_s = smp.steps_per_s(el / (args.steps * reps))
    line = {"metric": METRIC, "impl": "reference", "value": steps_per_s, "unit": "steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / steps_per_s, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_of(w, mode, args.layers, args.gpus),
            "cpu_baseline": {"value": steps_per_s, "unit": "steps/s", "cores": len(smp.slices),
                             "kind": "oracle",
                             "sample": smp.describe(args.steps * reps, el)},
            "e2e": {"value": steps_per_s, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def oracle_precision_map(w):
    """The decay-ranked map of a mixed workload from the whole run's gates."""
    import oracle
    from quantized_recurrent_state_decode_b200 import inputs as I
    pm = I.uniform_prec_map(w)
    if pm is not None:
        return pm.numpy()
    decay = I.decay_tensor(w)
    return oracle.precision_map(oracle.decay_means(decay.numpy()), I.n_int8_heads(w))


def config_of(w, mode, layers, n):
    from quantized_recurrent_state_decode_b200 import inputs as I
    prec = {"int8": "int8", "int4": "int4", "mixed": "mixed int8/int4"}[w.precision]
    return {"workload": w.name, "family": w.family, "batch_per_gpu": w.batch,
            "global_batch": w.batch * n, "heads": w.heads, "d_k": w.d_k, "d_v": w.d_v,
            "group": w.group, "state": prec,
            "rounding": {0: "rtn", 1: "sr", 2: "bdr"}[mode],
            "layers_rotated": layers,
            "l2": "inputs larger than L2: %d layer states rotated per step" % layers,
            "parallelism": "dp%d" % n}


# -------------------------------------------------------------------- GPU ---

def precision_map(w, lrs, dev):
    """Per-head precision: uniform for int8/int4 workloads; for mixed ones,
    the library's mean decay per head over the whole run's gates, ranked."""
    import numpy as np
    import torch
    from quantized_recurrent_state_decode_b200 import inputs as I
    pm = I.uniform_prec_map(w)
    if pm is not None:
        return pm.numpy()
    decay = I.decay_tensor(w, device=dev)
    outer, H, inner = decay.shape
    means = torch.zeros(H, dtype=torch.float64, device=dev)
    lrs.lrs_decay_head_means(decay, outer, H, inner, means)
    torch.cuda.synchronize()
    return lrs.lrs_precision_map(means.cpu().numpy(), I.n_int8_heads(w))


def state_bytes(w, pm=None):
    """Algorithmic bytes of one step: codes and scales, each read once and
    written once (per-head code widths from the precision map)."""
    G = w.d_k // w.group
    bits = [8] * w.heads if pm is None else [int(b) for b in pm]
    per_row = sum(w.d_k * w.d_v * b // 8 + G * w.d_v * 4 for b in bits)
    return 2 * w.batch * per_row


def run_gpu(args, w):
    import numpy as np
    import torch
    import torch.distributed as dist

    from quantized_recurrent_state_decode_b200 import inputs as I
    from quantized_recurrent_state_decode_b200 import lrs
    from quantized_recurrent_state_decode_b200.shard import batch_slice, max_over_ranks

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    mode = MODES[args.mode] if args.mode else w.mode

    # weak scaling: every rank owns a batch slice of size w.batch of a global
    # batch of w.batch * world rows
    wg = w.with_batch(w.batch * world)
    off, nb = batch_slice(wg.batch, rank, world)
    wl = w.with_batch(nb)
    pm = precision_map(w, lrs, dev)
    shp = lrs.shape(nb, w.heads, w.d_k, w.d_v, w.group, w.update_kind, w.gate_kind)
    L = args.layers
    states = [lrs.lrs_state_alloc(shp, pm) for _ in range(L)]
    S0 = I.initial_state(wg, off, nb, device=dev)
    for st in states:
        lrs.lrs_state_import_fp32(st, S0)
    del S0
    NI = 8
    xs = [I.step_inputs(wg, t, off, nb, device=dev) for t in range(NI)]
    out = torch.empty(nb, w.heads, w.d_v, device=dev)
    seed = I.sr_seed(w)
    torch.cuda.synchronize()
    # all work runs on one non-default stream (graph capture needs one)
    stream = torch.cuda.Stream()
    pick = lambda i: (states[i % L], xs[i % NI], i)

    with torch.cuda.stream(stream):
        for t in range(args.warmup):                    # warm-up, eager launches
            st, x, _ = pick(t)
            lrs.lrs_decode_step(st, st.state_codes, st.scales, st.prec_map, x["q"], x["k"],
                                x["v"], x["gates"], x["beta"], out, seed, t, mode, stream)
        lrs.lrs_sync(stream)
        # the timed steps: CUDA graphs of `chunk` launches, replayed
        chunk = min(args.steps, 64)
        full, rem = divmod(args.steps, chunk)
        g_chunk = _capture_on(stream, chunk, pick, lrs, out, seed, mode)
        g_rem = _capture_on(stream, rem, pick, lrs, out, seed, mode) if rem else None
        g_chunk.replay()                                # one untimed replay
        torch.cuda.synchronize()

        sampler = ClockSampler(local)
        if rank == 0:
            sampler.start()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_wall0 = time.time()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(full):
            g_chunk.replay()
        if g_rem is not None:
            g_rem.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        t_wall1 = time.time()
        if world > 1:
            dist.barrier()
    ms = ev0.elapsed_time(ev1)
    lrs.lrs_sync(stream)
    del g_chunk, g_rem
    ms_max = max_over_ranks(ms, device=dev)
    clocks = sampler.summary(t_wall0, t_wall1) if rank == 0 else None
    if rank == 0:
        sampler.stop()

    steps_per_s = world * args.steps / (ms_max / 1e3)
    bytes_step = state_bytes(wl, pm)
    launch_s = ms / 1e3 / args.steps
    achieved = bytes_step / launch_s / 1e9
    peak, peak_kind = measured_peaks()

    # end to end: host inputs in pinned memory, copies inside the timed region,
    # over at least 256 steps whatever --steps is (the host step overlaps
    # consecutive calls through two staging buffers: it needs a long run to
    # reach its steady state)
    e2e_steps = max(256, min(args.steps, 1024))
    xh = [{n: (None if v is None else v.cpu().pin_memory()) for n, v in x.items()} for x in xs]
    out_h = torch.empty(nb, w.heads, w.d_v).pin_memory()
    st0 = states[0]
    with torch.cuda.stream(stream):
        for t in range(min(args.warmup, 8)):
            x = xh[t % NI]
            lrs.lrs_decode_step_host(st0, x["q"], x["k"], x["v"], x["gates"], x["beta"], out_h,
                                     seed, t, mode, stream)
        lrs.lrs_sync(stream)
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for t in range(e2e_steps):
            st = states[t % L]
            x = xh[t % NI]
            lrs.lrs_decode_step_host(st, x["q"], x["k"], x["v"], x["gates"], x["beta"], out_h,
                                     seed, t, mode, stream)
        e1.record(stream)
        torch.cuda.synchronize()
    lrs.lrs_sync(stream)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device=dev)
    h2d = sum(v.numel() * 4 for v in xh[0].values() if v is not None)
    d2h = out_h.numel() * 4
    pinned = pinned_copy_rates(h2d, d2h, dev, stream)
    e2e_sps = world * e2e_steps / (e2e_ms / 1e3)

    extras = {}
    if not args.no_extras and rank == 0:
        with torch.cuda.stream(stream):
            extras = run_extras(args, w, wl, states, xs, out, seed, stream, L, NI, mode, dev, pm)

    for st in states:
        lrs.lrs_state_free(st)
    if args.configs and rank == 0:
        extras["configs"] = run_configs(dev, stream)
    if not args.no_extras and rank == 0 and args.drift_steps > 0:
        extras["drift"] = run_drift(dev, stream, args.drift_steps)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    line = {
        "metric": METRIC, "value": steps_per_s, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded draws with the workload's distributions)",
        "config": config_of(w, mode, L, world),
        "state_gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind + " (hbm_gbs, burst copy)",
                     "traffic": profiled_traffic(),
                     "algorithmic_bytes_per_launch": bytes_step,
                     "kernel": "lrs::step_kernel<C=%d,group=%d,%s,%s,%s>" % (
                         w.d_v // 32, w.group, "delta" if w.update_kind else "gated",
                         "per_key" if w.gate_kind else "scalar",
                         {0: "rtn", 1: "sr", 2: "bdr"}[mode])},
        "e2e": {"value": e2e_sps, "unit": "steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "h2d_gbs_achieved": e2e_sps / world * h2d / 1e9,
                "pinned_copy_gbs_measured": pinned,
                "api": "lrs_decode_step_host"},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    line.update(extras)
    if args.cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, mode)
    print(json.dumps(line))


def pinned_copy_rates(h2d, d2h, dev, stream, reps=16, trials=5):
    """Plain pinned-host <-> device copy rates at the step's own sizes (one
    host-to-device copy of h2d bytes, one device-to-host copy of d2h bytes),
    the ceiling of the host-buffer step's copies: the best of `trials` runs of
    `reps` back-to-back copies."""
    import torch
    hs = torch.empty(h2d // 4).pin_memory()
    ds = torch.empty(h2d // 4, device=dev)
    ho = torch.empty(d2h // 4).pin_memory()
    do = torch.empty(d2h // 4, device=dev)
    res = {}
    with torch.cuda.stream(stream):
        for name, dst, src, nbytes in (("h2d", ds, hs, h2d), ("d2h", ho, do, d2h)):
            dst.copy_(src, non_blocking=True)
            best = 0.0
            for _ in range(trials):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    dst.copy_(src, non_blocking=True)
                e1.record(stream)
                torch.cuda.synchronize()
                best = max(best, nbytes * reps / (e0.elapsed_time(e1) / 1e3) / 1e9)
            res[name] = best
    return res


def _capture_on(stream, n, pick, lrs, out, seed, mode):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            st, x, t = pick(i)
            lrs.lrs_decode_step(st, st.state_codes, st.scales, st.prec_map, x["q"], x["k"],
                                x["v"], x["gates"], x["beta"], out, seed, t, mode, stream)
    return g


def run_extras(args, w, wl, states, xs, out, seed, stream, L, NI, mode, dev, pm):
    """Other rounding modes on the same state, and the fp32-state kernel on the
    same inputs (rank 0 only, not part of the headline number)."""
    import torch
    from quantized_recurrent_state_decode_b200 import lrs
    res = {}
    n = 640
    for name, m in (("sr", 1), ("bdr", 2), ("rtn", 0)):
        if m == mode:
            continue
        for i in range(8):   # eager launches before capture
            st, x, t = states[i % L], xs[i % NI], i
            lrs.lrs_decode_step(st, st.state_codes, st.scales, st.prec_map, x["q"], x["k"],
                                x["v"], x["gates"], x["beta"], out, seed, t, m, stream)
        g = _capture_on(stream, n, lambda i: (states[i % L], xs[i % NI], i), lrs, out, seed, m)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / n
        res["mode_" + name] = {"ms_per_step": ms, "steps_per_s": 1e3 / ms,
                               "state_gbs": state_bytes(wl, pm) / (ms / 1e3) / 1e9}
        del g
    lrs.lrs_sync()
    # the same step with bfloat16 q, k, v and out
    xb = [{k: (v.to(torch.bfloat16) if k in ("q", "k", "v") else v) for k, v in x.items()}
          for x in xs]
    outb = torch.empty(out.shape, dtype=torch.bfloat16, device=dev)

    def step_bf16(i):
        st, x = states[i % L], xb[i % NI]
        lrs.lrs_decode_step_bf16(st, st.state_codes, st.scales, st.prec_map, x["q"], x["k"],
                                 x["v"], x["gates"], x["beta"], outb, seed, i, mode, stream)
    for i in range(8):
        step_bf16(i)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            step_bf16(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    io_f32 = sum(v.numel() * 4 for v in xs[0].values() if v is not None) + out.numel() * 4
    io_b = sum(v.numel() * v.element_size() for v in xb[0].values() if v is not None) + \
        outb.numel() * 2
    res["io_bf16"] = {"ms_per_step": ms, "steps_per_s": 1e3 / ms,
                      "state_gbs": state_bytes(wl, pm) / (ms / 1e3) / 1e9,
                      "io_bytes_per_step": io_b, "io_bytes_per_step_f32": io_f32,
                      "api": "lrs_decode_step_bf16"}
    del g
    lrs.lrs_sync()
    res["chunk"] = run_chunk_extra(w, wl, states, seed, stream, L, mode, dev, pm)
    res["lrb"] = run_lrb_extra(w, wl, states, xs, out, seed, stream, L, NI, mode, dev, pm)
    # fp32 state kernel: 4 rotated fp32 states
    shp = lrs.shape(wl.batch, w.heads, w.d_k, w.d_v, w.group, w.update_kind, w.gate_kind)
    Ls = 4
    Ss = [torch.zeros(wl.batch, w.heads, w.d_k, w.d_v, device=dev) for _ in range(Ls)]
    nf = 256
    for i in range(4):
        x = xs[i % NI]
        lrs.lrs_fp32_decode_step(shp, Ss[i % Ls], x["q"], x["k"], x["v"], x["gates"], x["beta"],
                                 out, stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(nf):
            x = xs[i % NI]
            lrs.lrs_fp32_decode_step(shp, Ss[i % Ls], x["q"], x["k"], x["v"], x["gates"],
                                     x["beta"], out, stream)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / nf
    fb = wl.batch * w.heads * w.d_k * w.d_v * 4 * 2
    res["fp32_state_kernel"] = {"ms_per_step": ms, "steps_per_s": 1e3 / ms,
                                "state_gbs": fb / (ms / 1e3) / 1e9, "bytes_per_step": fb}
    del g, Ss
    return res


# The five synthetic workloads the step is specified on, each in its stated
# rounding mode(s): (label, workload, batch override, modes).
CONFIG_RUNS = [
    ("C1", "gla_rtn_int8_b2h2_64", None, ("rtn",)),
    ("C2", "gdn_sr_int8_b64h16_128", None, ("sr",)),
    ("C3", "mamba2_mixed_sr_b128h64", None, ("sr",)),
    ("C4", "gla_bdr_int4_b256h32_128", None, ("bdr", "rtn")),
    ("C5", "gdn_mixed_sr_h32_128", 64, ("sr",)),
    ("C5", "gdn_mixed_sr_h32_128", 256, ("sr",)),
    ("C5", "gdn_mixed_sr_h32_128", 1024, ("sr",)),
]
L2_BYTES = 126 * 2**20


def _time_graph(stream, n, launch):
    """Device time per launch of n launches captured in one CUDA graph
    (eager warm-up launches first, one untimed replay)."""
    import torch
    for i in range(3):
        launch(i)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            launch(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    del g
    return ms


def run_configs(dev, stream, n=64):
    """Every specified workload in its rounding mode(s): the quantized step and
    the fp32-state kernel on the same inputs, each over layer states rotated so
    that their total is at least 4x the L2 (one state at most where a single
    state already exceeds that; the tiny first workload stays in L2)."""
    import torch
    from quantized_recurrent_state_decode_b200 import inputs as I
    from quantized_recurrent_state_decode_b200 import lrs
    peak, peak_kind = measured_peaks()
    rows = []
    for label, name, batch, modes in CONFIG_RUNS:
        w = I.WORKLOADS[name]
        if batch:
            w = w.with_batch(batch)
        pm = precision_map(w, lrs, dev)
        shp = lrs.shape(w.batch, w.heads, w.d_k, w.d_v, w.group, w.update_kind, w.gate_kind)
        sb = state_bytes(w, pm)
        L = max(1, min(64, -(-4 * L2_BYTES // (sb // 2))))
        states = [lrs.lrs_state_alloc(shp, pm) for _ in range(L)]
        S0 = I.initial_state(w, device=dev)
        for st in states:
            lrs.lrs_state_import_fp32(st, S0)
        NI = 8
        xs = [I.step_inputs(w, t, device=dev) for t in range(NI)]
        out = torch.empty(w.batch, w.heads, w.d_v, device=dev)
        seed = I.sr_seed(w)
        fb = w.batch * w.heads * w.d_k * w.d_v * 4 * 2          # fp32 state read + written
        Lf = max(1, min(16, -(-4 * L2_BYTES // (fb // 2))))
        Ss = [S0.clone() for _ in range(Lf)]
        del S0
        with torch.cuda.stream(stream):
            def f32(i):
                x = xs[i % NI]
                lrs.lrs_fp32_decode_step(shp, Ss[i % Lf], x["q"], x["k"], x["v"], x["gates"],
                                         x["beta"], out, stream)
            ms_f = _time_graph(stream, n, f32)
            for mname in modes:
                m = MODES[mname]

                def step(i, m=m):
                    st, x = states[i % L], xs[i % NI]
                    lrs.lrs_decode_step(st, st.state_codes, st.scales, st.prec_map, x["q"],
                                        x["k"], x["v"], x["gates"], x["beta"], out, seed, i, m,
                                        stream)
                ms = _time_graph(stream, n, step)
                lrs.lrs_sync(stream)
                gbs = sb / (ms / 1e3) / 1e9
                rows.append({
                    "config": label, "workload": w.name, "family": w.family, "batch": w.batch,
                    "heads": w.heads, "d_k": w.d_k, "d_v": w.d_v, "group": w.group,
                    "state": w.precision, "rounding": mname,
                    "us_per_step": ms * 1e3, "steps_per_s": 1e3 / ms,
                    "state_bytes_per_step": sb, "state_gbs": gbs, "hbm_frac": gbs / peak,
                    "layers_rotated": L,
                    "fp32_state_kernel": {"us_per_step": ms_f * 1e3, "bytes_per_step": fb,
                                          "state_gbs": fb / (ms_f / 1e3) / 1e9,
                                          "hbm_frac": fb / (ms_f / 1e3) / 1e9 / peak,
                                          "layers_rotated": Lf},
                    "speedup_vs_fp32_state": ms_f / ms})
                # the NEXT rows on the same states and inputs, in the same mode
                rows[-1]["lrb"] = run_lrb_extra(w, w, states, xs, out, seed, stream, L, NI, m,
                                                dev, pm)
                rows[-1]["chunk"] = run_chunk_extra(w, w, states, seed, stream, L, m, dev, pm)
        for st in states:
            lrs.lrs_state_free(st)
        del Ss, xs, out
        torch.cuda.empty_cache()
    return {"peak_gbs": peak, "peak_kind": peak_kind, "timed_launches": n,
            "timing": "CUDA events around a graph of %d launches; state bytes = codes + "
                      "scales read and written once" % n, "runs": rows}


FP32_LANES_PER_SM = 128      # fp32 fused multiply-add lanes per SM (sm_100)


def run_chunk_extra(w, wl, states, seed, stream, L, mode, dev, pm, T=16, n=32):
    """The multi-token update (T tokens per tile, one requantization) on the
    same states: time per chunk, and its fp32 arithmetic against the fp32 FMA
    peak at the SM clock limit (the chunk is bound by arithmetic, not HBM)."""
    import torch
    from quantized_recurrent_state_decode_b200 import inputs as I
    from quantized_recurrent_state_decode_b200 import lrs
    if w.d_k not in (64, 128) or w.d_v not in (64, 128):
        return None
    xc = I.chunk_inputs(wl, 0, T, device=dev)
    out = torch.empty(T, wl.batch, w.heads, w.d_v, device=dev)

    def launch(i):
        st = states[i % L]
        lrs.lrs_chunk_step(st, st.state_codes, st.scales, st.prec_map, T, xc["q"], xc["k"],
                           xc["v"], xc["gates"], xc["beta"], out, seed, i, mode, stream)
    for i in range(4):
        launch(i)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            launch(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    del g
    lrs.lrs_sync()
    elems = wl.batch * w.heads * w.d_k * w.d_v
    flops_el = 7 if w.update_kind == 1 else 5       # k*w, g*x + kw, q*x (+ k*x for u)
    flops = elems * T * flops_el
    props = torch.cuda.get_device_properties(dev)
    clk = _sm_max_mhz()
    peak = props.multi_processor_count * FP32_LANES_PER_SM * 2 * clk * 1e6 / 1e12 if clk else None
    achieved = flops / (ms / 1e3) / 1e12
    io = sum(v.numel() * 4 for v in xc.values() if v is not None) + out.numel() * 4
    return {"tokens_per_chunk": T, "ms_per_chunk": ms,
            "tile_tokens_per_s": wl.batch * w.heads * T / (ms / 1e3),
            "api": "lrs_chunk_step",
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak if peak else None,
                         "peak_kind": "fp32 FMA lanes x 2 x SMs x max SM clock (%s MHz)" % clk,
                         "flops_per_element_token": flops_el},
            "state_bytes": state_bytes(wl, pm),
            "io_bytes_per_chunk": io}


def run_lrb_extra(w, wl, states, xs, out, seed, stream, L, NI, mode, dev, pm, rank=4, n=64):
    """The decode step with a Low-Rank Bypass buffer of rank `rank` on the same
    states and inputs (one buffer per layer state; n steps cover n/rank merges).
    Algorithmic bytes per step: the state's codes and scales read and written,
    plus the buffer rows read (filled components) and written (filled + the new
    one), averaged over the rank-step cycle: rank * (d_k + d_v) * 4 per tile."""
    import torch
    from quantized_recurrent_state_decode_b200 import lrs
    if w.d_k not in (64, 128) or w.d_v not in (64, 128):
        return None
    Us = [torch.zeros(wl.batch, w.heads, rank, w.d_k, device=dev) for _ in range(L)]
    Vs = [torch.zeros(wl.batch, w.heads, rank, w.d_v, device=dev) for _ in range(L)]

    def launch(i):
        st, x = states[i % L], xs[i % NI]
        lrs.lrs_lrb_step(st, st.state_codes, st.scales, st.prec_map, rank, Us[i % L], Vs[i % L],
                         x["q"], x["k"], x["v"], x["gates"], x["beta"], out, seed, i // L, mode,
                         stream)
    for i in range(L * rank):
        launch(i)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            launch(i + L * rank)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    del g
    lrs.lrs_sync()
    tiles = wl.batch * w.heads
    nbytes = state_bytes(wl, pm) + tiles * rank * (w.d_k + w.d_v) * 4
    peak, peak_kind = measured_peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"rank": rank, "ms_per_step": ms, "steps_per_s": 1e3 / ms, "api": "lrs_lrb_step",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "algorithmic_bytes_per_launch": nbytes}}


DRIFT_WORKLOAD = "gla_bdr_int4_b256h32_128"


def run_drift(dev, stream, steps=1024, batch=None):
    """Output drift of the int4 GLA workload against the fp32-state kernel on
    the same inputs: e_t = ||o_q - o_fp32||_2 / ||o_fp32||_2 over every
    (b, h, j) of step t, at t = 1, 2, 4, ..., for round to nearest, bounded
    directional rounding, stochastic rounding and the rank-4 Low-Rank Bypass
    with RTN and with BDR. Every variant starts from the same state and reads
    the same inputs; the norms are taken after the step, outside any timing."""
    import torch
    from quantized_recurrent_state_decode_b200 import inputs as I
    from quantized_recurrent_state_decode_b200 import lrs
    w = I.WORKLOADS[DRIFT_WORKLOAD]
    if batch:
        w = w.with_batch(batch)
    pm = I.uniform_prec_map(w).numpy()
    shp = lrs.shape(w.batch, w.heads, w.d_k, w.d_v, w.group, w.update_kind, w.gate_kind)
    seed = I.sr_seed(w)
    rank = 4
    variants = [("rtn", I.ROUND_RTN, 0), ("bdr", I.ROUND_BDR, 0), ("sr", I.ROUND_SR, 0),
                ("lrb4_rtn", I.ROUND_RTN, rank), ("lrb4_bdr", I.ROUND_BDR, rank)]
    S0 = I.initial_state(w, device=dev)
    S = S0.clone()
    states, bufs, outs = {}, {}, {}
    try:
        for name, _, r in variants:
            st = lrs.lrs_state_alloc(shp, pm)
            states[name] = st
            lrs.lrs_state_import_fp32(st, S0)
            if r:
                bufs[name] = (torch.zeros(w.batch, w.heads, r, w.d_k, device=dev),
                              torch.zeros(w.batch, w.heads, r, w.d_v, device=dev))
            outs[name] = torch.empty(w.batch, w.heads, w.d_v, device=dev)
        del S0
        of = torch.empty(w.batch, w.heads, w.d_v, device=dev)
        samples = [1 << i for i in range(steps.bit_length()) if (1 << i) <= steps]
        series = {name: [] for name, _, _ in variants}
        with torch.cuda.stream(stream):
            for t in range(steps):
                x = I.step_inputs(w, t, device=dev)
                lrs.lrs_fp32_decode_step(shp, S, x["q"], x["k"], x["v"], x["gates"], x["beta"],
                                         of, stream)
                for name, mode, r in variants:
                    st = states[name]
                    if r:
                        U, V = bufs[name]
                        lrs.lrs_lrb_step(st, st.state_codes, st.scales, st.prec_map, r, U, V,
                                         x["q"], x["k"], x["v"], x["gates"], x["beta"],
                                         outs[name], seed, t, mode, stream)
                    else:
                        lrs.lrs_decode_step(st, st.state_codes, st.scales, st.prec_map, x["q"],
                                            x["k"], x["v"], x["gates"], x["beta"], outs[name],
                                            seed, t, mode, stream)
                if t + 1 in samples:
                    ref = torch.linalg.vector_norm(of)
                    for name, _, _ in variants:
                        series[name].append(
                            (torch.linalg.vector_norm(outs[name] - of) / ref).item())
        lrs.lrs_sync(stream)
    finally:
        for st in states.values():
            lrs.lrs_state_free(st)
    res = {"workload": w.name, "batch": w.batch, "state": "int4", "group": w.group,
           "lrb_rank": rank,
           "measure": "||o_q - o_fp32||_2 / ||o_fp32||_2 over all (b, h, j) of step t",
           "reference": "lrs_fp32_decode_step on the same inputs", "t": samples}
    res.update(series)
    return res


def _sm_max_mhz():
    try:
        out = subprocess.run(["nvidia-smi", "--query-gpu=clocks.max.sm", "--format=csv,noheader,"
                              "nounits", "-i", os.environ.get("LOCAL_RANK", "0")],
                             capture_output=True, text=True, timeout=20).stdout
        return float(out.strip().splitlines()[0])
    except Exception:
        return None


def cpu_baseline(w, mode):
    """The oracle on the host cores, the same sampler as `--impl reference`,
    for about 12 s of oracle time."""
    smp = OracleSampler(w, mode)
    smp.step(0)
    el, steps = 0.0, 0
    while el < 12.0:
        el += smp.step(steps)
        steps += 1
    smp.close()
    return {"value": smp.steps_per_s(el / steps), "unit": "steps/s", "cores": len(smp.slices),
            "kind": "oracle", "sample": smp.describe(steps, el)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6400)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", default="lrs", choices=["lrs", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--mode", default=None, choices=sorted(MODES))
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--drift-steps", type=int, default=1024,
                    help="steps of the int4 output-drift series (0: skip it)")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the per-workload table (the `configs` key)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from quantized_recurrent_state_decode_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_batch(args.batch)
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        run_reference(args, w)
        return
    run_gpu(args, w)


if __name__ == "__main__":
    main()
