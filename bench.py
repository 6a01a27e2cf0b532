"""StreamKL benchmark: one step = the whole hot path on one batch of synthetic input:
forward (KL, LSE1, LSE2) + backward with P1 fixed (dQ2, dK2) + backward with P2 fixed
(dQ1, dK1), on the headline workload B=1, H=32, NQ=NK=16384, d=128, causal, shared keys,
bf16 inputs (Q1 ~ N(0,1), Q2 = 0.8 Q1 + 0.6 N(0,1), K ~ N(0,1), seeded).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  value = whole-job TFLOP/s over all ranks, with FLOPs counted
as 4d per unmasked (row, key) pair for the forward and 8d for each backward, causal pairs
halved.  With N > 1 (torchrun, one process per GPU) every rank runs its own batch of the
same workload (weak scaling, no data-path collective); timing is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (a bounded
sample of rows per step, rank 0 only).
"""
import argparse
import json
import math
import os
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd/bwd TFLOP/s & ms, H=32 N=16K d=128 causal bf16; % of B200 dense peak"
UNIT = "TFLOP/s"
WORKLOAD = "headline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0
L2_BYTES = 126 * 2**20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ------------------------------------------------------------------ multi-rank host logic
def rank_workload(base, rank):
    """Weak scaling: every rank gets its own batch of the same workload (own seed)."""
    from attention_kl_divergence_02_b200 import inputs
    return inputs.variant(base, seed=base.seed + 1000 * rank)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of timings over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    x = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(x, op=dist.ReduceOp.MAX)
    return x.tolist()


def job_tflops(world, flops_per_rank_step, ms_per_step):
    """Whole-job throughput: every rank's work divided by the slowest rank's time."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ roofline bookkeeping
# Share of the forward's exponentials that the kernel evaluates with the FMA-pipe polynomial
# instead of the exponential unit: 4 of the 16 column pairs of every 32-column chunk, for S1
# and for S2 (the kEmu1 / kEmu2 masks of the forward kernel).
FWD_POLY_SHARE = 0.25


def choose_peak(peaks, peak_src, timed_s, clk):
    """The bf16 denominator of a tensor-bound call: the burst figure when the timed region is
    short (under a second) and the sampled SM clock stayed at its maximum -- the conditions
    the burst GEMM was measured in -- else the sustained figure (a seconds-long loop under
    the power cap).  Returns (peak, label, reason)."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    clk = clk or {}
    mx = clk.get("sm_max_mhz") or peaks.get("sm_max_mhz")
    eff = clk.get("sm_mhz_effective")
    med, what = (eff, "effective SM clock (clock probe)") if eff else (
        clk.get("sm_mhz"), "median sampled SM clock")
    at_max = med is not None and mx is not None and med >= 0.97 * mx
    if timed_s < 1.0 and at_max:
        return burst, "%s bf16_tflops (burst)" % peak_src, (
            "timed region %.2f s < 1 s and %s %.0f MHz at its maximum %.0f"
            % (timed_s, what, med, mx))
    why = []
    if timed_s >= 1.0:
        why.append("timed region %.2f s >= 1 s" % timed_s)
    if not at_max:
        why.append("%s %s MHz below its maximum %s (power cap)" % (
            what, "%.0f" % med if med is not None else None, mx))
    return sus, "%s bf16_tflops_sustained" % peak_src, "; ".join(why)


def measure_exp_rates(binding, stream, gpu_index, target_ms=120.0):
    """Throughput of the two exponential paths (library probe: MUFU ex2.approx, and the
    FMA-pipe polynomial), each timed alone with CUDA events over ~target_ms, best of three,
    with the SM clock sampled meanwhile.  Returns exponentials per SM per clock for each
    path, with the clock and the raw rate they come from."""
    import torch
    sms = binding.streamkl_num_sms()
    out = {}
    clocks = ClockSampler(gpu_index, tag="exp")
    clocks.start()
    time.sleep(0.3)
    for kind, name in ((0, "mufu_ex2"), (1, "fma_poly")):
        def run(iters):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            rc, n = binding.streamkl_probe_exp2(kind, iters, stream)
            b.record(stream)
            torch.cuda.synchronize()
            if rc != binding.OK:
                raise RuntimeError("exp2 probe: %s" % binding.status_string(rc))
            return a.elapsed_time(b), n
        run(64)
        ms, _ = run(2000)
        iters = max(2000, int(2000 * target_ms / max(ms, 1e-3)))
        best = None
        for _ in range(3):
            ms, n = run(iters)
            rate = n / (ms * 1e-3)
            best = rate if best is None or rate > best else best
        out[name] = {"exps_per_s": best, "iters": iters}
    clk = clocks.stop()
    mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0
    for v in out.values():
        v["per_sm_per_clk"] = v["exps_per_s"] / (sms * mhz * 1e6)
        v["sm_mhz"] = mhz
    out["sms"] = sms
    out["clocks"] = clk
    return out


def exp_roofline(w, fwd_ms, rates, step_mhz):
    """The forward's exponential-unit roof: 2 exponentials per unmasked pair (causal pairs
    halved, as for the FLOPs), of which (1 - FWD_POLY_SHARE) run on the exponential unit; at
    the measured MUFU rate per SM per clock and the step's median SM clock, the shortest
    time that unit allows, divided by the forward's measured time."""
    exps = 2.0 * w.pairs()
    mufu = rates["mufu_ex2"]["per_sm_per_clk"] * rates["sms"] * step_mhz * 1e6   # exps / s
    poly = rates["fma_poly"]["per_sm_per_clk"] * rates["sms"] * step_mhz * 1e6
    t_mufu = (1.0 - FWD_POLY_SHARE) * exps / mufu
    return {"bound": "exp", "unit": "exp2/s", "exps_per_call": exps,
            "achieved": exps / (fwd_ms * 1e-3), "mufu_share": 1.0 - FWD_POLY_SHARE,
            "mufu_peak": mufu, "poly_peak": poly,
            "mufu_per_sm_per_clk": rates["mufu_ex2"]["per_sm_per_clk"],
            "poly_per_sm_per_clk": rates["fma_poly"]["per_sm_per_clk"],
            "frac": t_mufu * 1e3 / fwd_ms,
            "t_mufu_ms": t_mufu * 1e3, "t_all_on_mufu_ms": exps / mufu * 1e3,
            "note": "frac = time the exponential unit needs for its share of the forward's "
                    "exponentials at the measured rate and the step's median clock / forward time"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, tag="step"):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(),
                                 "streamkl_clocks_%s_rank%d.csv" % (tag, gpu_index))

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, power = [], None, set(), []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    clk, mx = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                smax = mx
                try:
                    power.append(float(parts[3]))
                except ValueError:
                    pass
                sm.append(clk)
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        loaded = [c for c in sm if smax and c > 0.3 * smax] or sm
        loaded.sort()
        med = loaded[len(loaded) // 2] if loaded else None
        return {"sm_mhz": med, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


class ClockProbe:
    """Effective SM clock over the timed region, from the library's clock probe: one warp on
    a stream of its own, beside the timed kernels, records (ns, SM cycles) every 50 us.
    Under the board's power cap the SM clock drops while the step runs, and the 100 ms
    nvidia-smi samples can miss it; cycles over nanoseconds cannot."""

    INTERVAL_NS = 50_000

    def __init__(self, binding, device):
        import torch
        self.binding, self.torch, self.device = binding, torch, device
        self.samples = None

    def start(self, expected_ms):
        torch = self.torch
        dur_ns = int(min(9.0e9, max(2.0e6, expected_ms * 1.5e6 + 20e6)))
        pairs = min(400_000, dur_ns // self.INTERVAL_NS + 16)
        self.samples = torch.zeros(2 + 2 * pairs, dtype=torch.int64, device=self.device)
        self.stream = torch.cuda.Stream(device=self.device)
        rc = self.binding.streamkl_probe_clock(dur_ns, self.INTERVAL_NS, self.samples, self.stream)
        if rc != self.binding.OK:
            raise RuntimeError("clock probe: %s" % self.binding.status_string(rc))

    def stop(self, region_ms):
        """Waits for the probe; returns the clock over its first region_ms milliseconds."""
        self.torch.cuda.synchronize()
        h = self.samples.cpu().tolist()
        n = int(h[0])
        t = [h[2 + 2 * i] for i in range(n)]
        c = [h[3 + 2 * i] for i in range(n)]
        if n < 2:
            return None
        last = max(i for i in range(n) if t[i] - t[0] <= region_ms * 1e6) if n else 0
        if last < 1:
            return None
        per = sorted((c[i + 1] - c[i]) / (t[i + 1] - t[i]) * 1e3 for i in range(last)
                     if t[i + 1] > t[i])
        return {"sm_mhz_effective": (c[last] - c[0]) / (t[last] - t[0]) * 1e3,
                "sm_mhz_effective_p10": per[len(per) // 10] if per else None,
                "sm_mhz_effective_p90": per[(9 * len(per)) // 10] if per else None,
                "pairs": last + 1, "span_ms": (t[last] - t[0]) * 1e-6,
                "how": "library clock probe beside the timed kernels: SM cycles (clock64) over "
                       "globaltimer ns every 50 us, first %.1f ms" % region_ms}


# ------------------------------------------------------------------ CPU oracle legs
def oracle_sample(w, n_rows, seed=0):
    """Bounded oracle sample of one step: forward + both backward settings for ``n_rows``
    random query rows of the workload (each row against all of its valid keys).  Returns
    (seconds, flops) with FLOPs of the oracle's own work: 4d per pair for the forward and
    6d per pair per backward row (recompute 4d + dQ 2d; the dK share of those rows is not
    formed)."""
    import numpy as np
    import oracle
    from attention_kl_divergence_02_b200 import inputs

    t = _host_inputs(w)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(w.B * w.Hq * w.NQ, size=n_rows, replace=False))
    i = rows % w.NQ
    pairs = float(np.sum(np.minimum(i + 1, w.NK) if w.causal else np.full(n_rows, w.NK)))
    t0 = time.perf_counter()
    oracle.fwd_rows(t["q1"], t["k1"], t["q2"], t["k2"], rows, scale=w.scale, causal=w.causal)
    for mode in (1, 2):
        oracle.bwd_dq_rows(mode, t["q1"], t["k1"], t["q2"], t["k2"], t["dkl"], rows,
                           scale=w.scale, causal=w.causal)
    dt = time.perf_counter() - t0
    return dt, pairs * w.d * (4 + 6 + 6)


_HOST = {}


def _host_inputs(w):
    from attention_kl_divergence_02_b200 import inputs
    if w.name not in _HOST:
        t = inputs.make(w, device="cpu")
        _HOST[w.name] = {k: inputs.to_f64(v) for k, v in t.items()}
    return _HOST[w.name]


def cpu_baseline(w, target_s=15.0):
    """Time the oracle on ~target_s seconds of sampled rows; TFLOP/s of that sample."""
    import oracle
    oracle.build()
    cores = oracle.num_threads()
    _host_inputs(w)
    total_rows = w.B * w.Hq * w.NQ
    n = max(8, 2 * cores)
    dt, flops = oracle_sample(w, n, seed=1)
    # grow the sample until it takes at least 2/3 of the target (small probes overstate the
    # per-row cost: too few rows per thread)
    for it in range(4):
        if dt >= 0.66 * target_s or n >= total_rows:
            break
        n = int(min(total_rows, max(n + 1, n * target_s / max(dt, 1e-3))))
        dt, flops = oracle_sample(w, n, seed=2 + it)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "%d random query rows of the %s workload (all their valid keys): forward "
                      "+ both backward settings (dQ rows) in the fp64 C oracle, OpenMP over rows; "
                      "%.1f s" % (n, w.name, dt)}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from attention_kl_divergence_02_b200 import inputs
    import oracle
    oracle.build()
    w = inputs.WORKLOADS[WORKLOAD]
    cores = oracle.num_threads()
    _host_inputs(w)
    # size the per-step sample so that warmup + steps take about two minutes
    dt, _ = oracle_sample(w, max(8, 2 * cores), seed=99)
    per_row = dt / max(8, 2 * cores)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = max(cores, int(budget / max(per_row, 1e-6)))
    for s in range(args.warmup):
        oracle_sample(w, n, seed=1000 + s)
    times, flops = [], 0.0
    for s in range(args.steps):
        dts, f = oracle_sample(w, n, seed=s)
        times.append(dts)
        flops += f
    total = sum(times)
    value = flops / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "B1 H32 NQ=NK=16384 d128 causal shared-K (headline)",
                   "sample_rows_per_step": n, "global_batch": 1, "seq_len": w.NQ},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "%d random query rows per step: forward + both backward "
                                   "settings (dQ rows), fp64 C oracle" % n},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_gpu(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from attention_kl_divergence_02_b200 import binding, inputs

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    binding.load()
    base = inputs.WORKLOADS[WORKLOAD]
    if args.heads != base.Hq:  # reduced-head case for profiler captures only
        base = inputs.variant(base, Hq=args.heads, Hkv=args.heads)
    w = rank_workload(base, rank)
    t = inputs.make(w, device=dev)
    B, Hq, NQ, d = w.B, w.Hq, w.NQ, w.d
    stream = torch.cuda.current_stream()
    kl, l1, l2 = (torch.empty((B, Hq, NQ), device=dev) for _ in range(3))
    g = {m: (torch.empty_like(t["q1"]), torch.empty_like(t["k1"])) for m in (1, 2)}
    ws = torch.empty(binding.streamkl_bwd_workspace_bytes(B, Hq, w.Hkv, NQ, w.NK, d) // 4, device=dev)

    # NVTX ranges name each call for a timeline profiler (host-side markers only)
    def fwd():
        torch.cuda.nvtx.range_push("streamkl_fwd")
        binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal,
                    out=(kl, l1, l2), stream=stream)
        torch.cuda.nvtx.range_pop()

    def bwd(mode):
        torch.cuda.nvtx.range_push("streamkl_bwd_mode%d" % mode)
        binding.bwd(mode, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], scale=w.scale,
                    causal=w.causal, out=g[mode], workspace=ws, stream=stream)
        torch.cuda.nvtx.range_pop()

    def barrier():
        if world > 1:
            dist.barrier()

    wa, wb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(args.warmup):
        if i == args.warmup - 1:
            wa.record(stream)
        fwd(); bwd(1); bwd(2)
    wb.record(stream)
    torch.cuda.synchronize()
    warm_step_ms = wa.elapsed_time(wb)
    st = binding.streamkl_device_status()
    if st != binding.OK:
        raise RuntimeError("device status after warm-up: %s" % binding.status_string(st))

    # ---- timed region: K steps, events between the three calls of every step
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    probe = ClockProbe(binding, dev)
    barrier()
    torch.cuda.synchronize()
    probe.start(warm_step_ms * args.steps)
    t_start.record(stream)
    for k in range(args.steps):
        ev[k][0].record(stream)
        fwd()
        ev[k][1].record(stream)
        bwd(1)
        ev[k][2].record(stream)
        bwd(2)
        ev[k][3].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    region_ms = t_start.elapsed_time(t_end)
    eff = probe.stop(region_ms)
    if eff:
        clk.update(eff)
    st = binding.streamkl_device_status()
    if st != binding.OK:
        raise RuntimeError("device status after the timed region: %s" % binding.status_string(st))
    total_ms = region_ms
    f_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    b1_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    b2_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    total_ms, f_ms, b1_ms, b2_ms = max_over_ranks([total_ms, f_ms, b1_ms, b2_ms], device=dev)
    ms_step = total_ms / args.steps
    step_flops = w.fwd_flops() + 2 * w.bwd_flops()
    value = job_tflops(world, step_flops, ms_step)

    # ---- end to end through the public API with host buffers (pinned), copies timed.  Every
    # step copies its own inputs host -> device and reads its result (KL and both LSEs per
    # row, the loss the step produces) device -> host; the gradients stay on the device for
    # the optimiser.  The copy of step k+2's inputs runs on a second stream into the other of
    # two device buffers while the steps before it compute, and step k's result is read back
    # on a third stream, from the other of two device result buffers, while step k+1
    # computes; events order every buffer's reuse, and the region ends after the last read.
    e2e = None
    if not args.skip_e2e:
        hin = {k: v.cpu().pin_memory() for k, v in inputs.make(w, device="cpu").items()}
        names = [k for k in hin if k != "k2" or not w.shared_k]
        dbuf = [{k: torch.empty_like(hin[k], device=dev) for k in names} for _ in range(2)]
        hout = [{"kl": torch.empty((B, Hq, NQ), pin_memory=True),
                 "lse1": torch.empty((B, Hq, NQ), pin_memory=True),
                 "lse2": torch.empty((B, Hq, NQ), pin_memory=True)} for _ in range(2)]
        h2d = sum(hin[k].numel() * hin[k].element_size() for k in names)
        d2h = sum(v.numel() * v.element_size() for v in hout[0].values())
        copy_stream = torch.cuda.Stream(device=dev)
        read_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        consumed = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        read = [torch.cuda.Event() for _ in range(2)]
        res = [tuple(torch.empty((B, Hq, NQ), device=dev) for _ in range(3)) for _ in range(2)]

        def h2d_copy(slot):
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(consumed[slot])       # the buffer's last reader is done
                for k in names:
                    dbuf[slot][k].copy_(hin[k], non_blocking=True)
                copied[slot].record(copy_stream)

        def e2e_step(k, n_total):
            slot = k & 1
            stream.wait_event(copied[slot])
            stream.wait_event(read[slot])                     # step k-2's result is on the host
            x = dbuf[slot]
            k2 = x["k1"] if w.shared_k else x["k2"]
            rkl, rl1, rl2 = res[slot]
            binding.fwd(x["q1"], x["k1"], x["q2"], k2, scale=w.scale, causal=w.causal,
                        out=(rkl, rl1, rl2), stream=stream)
            for m in (1, 2):
                binding.bwd(m, x["q1"], x["k1"], x["q2"], k2, rkl, rl1, rl2, x["dkl"],
                            scale=w.scale, causal=w.causal, out=g[m], workspace=ws, stream=stream)
            consumed[slot].record(stream)
            computed[slot].record(stream)
            if k + 2 < n_total:
                h2d_copy(slot)                                # inputs of step k+2
            with torch.cuda.stream(read_stream):
                read_stream.wait_event(computed[slot])
                o = hout[slot]
                o["kl"].copy_(rkl, non_blocking=True)
                o["lse1"].copy_(rl1, non_blocking=True)
                o["lse2"].copy_(rl2, non_blocking=True)
                read[slot].record(read_stream)

        def e2e_run(n):
            for ev_ in consumed + read:
                ev_.record(stream)
            h2d_copy(0)
            if n > 1:
                h2d_copy(1)
            for k in range(n):
                e2e_step(k, n)

        e2e_run(2)
        torch.cuda.synchronize()
        ne = max(3, args.steps)   # as many steps as the device region; the first copy is not hidden
        barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        e_probe = ClockProbe(binding, dev)
        e_probe.start(ms_step * ne * 1.2)
        a.record(stream)
        e2e_run(ne)
        stream.wait_stream(copy_stream)
        stream.wait_stream(read_stream)
        b.record(stream)
        torch.cuda.synchronize()
        e_region = a.elapsed_time(b)
        e_eff = e_probe.stop(e_region)
        e_ms = max_over_ranks([e_region / ne], device=dev)[0]
        e2e = {"value": job_tflops(world, step_flops, e_ms), "unit": UNIT,
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "sm_mhz_effective": e_eff["sm_mhz_effective"] if e_eff else None,
               "note": "public API with pinned host buffers; each step copies its own inputs in "
                       "(overlapped with the previous step's compute on a second stream) and "
                       "reads its result (KL, LSE1, LSE2) back (overlapped with the next step's "
                       "compute on a third stream; the region ends after the last read); as many steps as the "
                       "device region, the first step's input copy not hidden"}

    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak, peak_label, peak_reason = choose_peak(peaks, peak_src, total_ms * 1e-3, clk)
    calls = {"fwd": (f_ms, w.fwd_flops()), "bwd_mode1": (b1_ms, w.bwd_flops()),
             "bwd_mode2": (b2_ms, w.bwd_flops())}
    tflops = {k: fl / (ms * 1e-3) / 1e12 for k, (ms, fl) in calls.items()}
    dom = max(calls, key=lambda k: calls[k][0])
    achieved = tflops[dom]
    traffic = load_traffic(dom)
    exp_roof = None
    if not args.skip_exp:
        rates = measure_exp_rates(binding, stream, local)
        step_mhz = clk.get("sm_mhz_effective") or clk.get("sm_mhz") or rates["mufu_ex2"]["sm_mhz"]
        exp_roof = exp_roofline(w, f_ms, rates, step_mhz)
        exp_roof["probe_clocks"] = rates["clocks"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "B1 H%d NQ=NK=16384 d128 causal shared-K (%s); step = "
                               "forward + backward P1-fixed + backward P2-fixed"
                               % (Hq, "headline" if Hq == 32 else "reduced heads"),
                   "global_batch": world * B, "seq_len": NQ, "heads": Hq, "head_dim": d,
                   "parallelism": "dp%d (independent batch per GPU, no collective)" % world,
                   "l2": "inputs (3 x 128 MiB bf16) larger than the 126 MB L2; no flush"},
        "fwd_ms": f_ms, "fwd_tflops": tflops["fwd"],
        "bwd_mode1_ms": b1_ms, "bwd_mode1_tflops": tflops["bwd_mode1"],
        "bwd_mode2_ms": b2_ms, "bwd_mode2_tflops": tflops["bwd_mode2"],
        "pct_of_peak": {"fwd": 100 * tflops["fwd"] / burst,
                        "bwd_mode1": 100 * tflops["bwd_mode1"] / burst,
                        "bwd_mode2": 100 * tflops["bwd_mode2"] / burst,
                        "step": 100 * value / world / burst,
                        "basis": "%s bf16 %.1f TFLOP/s (burst); nominal dense %.0f gives fwd %.1f%%"
                                 % (peak_src, burst, NOMINAL_BF16_TFLOPS,
                                    100 * tflops["fwd"] / NOMINAL_BF16_TFLOPS)},
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "fwd_frac": tflops["fwd"] / peak, "bwd_mode1_frac": tflops["bwd_mode1"] / peak,
                     "bwd_mode2_frac": tflops["bwd_mode2"] / peak,
                     "peak_source": peak_label, "peak_rule": peak_reason,
                     "peak_burst": burst, "frac_of_burst": achieved / burst,
                     "peak_sustained": float(peaks.get("bf16_tflops_sustained",
                                                       FALLBACK_PEAKS["bf16_tflops_sustained"])),
                     "note": "achieved = algorithmic FLOPs per call / CUDA-event duration of the "
                             "call on its stream%s" % (
                                 "; the backward call also runs the workspace memset and the "
                                 "dK convert kernel" if dom.startswith("bwd") else "")},
        "exp_roofline": exp_roof,
        "clocks": clk,
        "gpu_launches": 5 * args.steps + (1 if eff else 0),
        "e2e": e2e,
    }
    if world == 1 and rank == 0 and not args.skip_cpu:
        line["cpu_baseline"] = cpu_baseline(base)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_decode(args):
    """Split-K forward on the decode workload (one query row per head, 131072 keys): bound by
    streaming the keys from HBM, so it reports GB/s of algorithmic traffic against the
    measured copy bandwidth, and the unsplit forward beside it."""
    import torch

    from attention_kl_divergence_02_b200 import binding, inputs

    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--decode measures one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    binding.load()
    w = inputs.WORKLOADS["decode"]
    t = inputs.make(w, device=dev)
    B, Hq, NQ, NK, d = w.B, w.Hq, w.NQ, w.NK, w.d
    splits = binding.streamkl_fwd_splits(B, Hq, NQ, NK)
    need = binding.streamkl_fwd_splitk_workspace_bytes(B, Hq, NQ, NK, 0)
    ws = torch.empty(max(4, need) // 4, dtype=torch.float32, device=dev)
    out = tuple(torch.empty((B, Hq, NQ), device=dev) for _ in range(3))
    stream = torch.cuda.current_stream()

    def split():
        binding.fwd_splitk(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal,
                           splits=0, out=out, workspace=ws, stream=stream)

    def unsplit():
        binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal, out=out,
                    stream=stream)

    for _ in range(args.warmup):
        split()
        unsplit()
    torch.cuda.synchronize()
    st = binding.streamkl_device_status()
    if st != binding.OK:
        raise RuntimeError("device status after warm-up: %s" % binding.status_string(st))

    def timed(fn):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    s_ms = timed(split)
    u_ms = timed(unsplit)
    clk = clocks.stop()
    st = binding.streamkl_device_status()
    if st != binding.OK:
        raise RuntimeError("device status after the timed region: %s" % binding.status_string(st))
    # algorithmic bytes: Q1, Q2, the keys once (shared), 12 bytes of output per row
    rows = B * Hq * NQ
    nbytes = 2 * rows * d * 2 + B * w.Hkv * NK * d * 2 * (1 if w.shared_k else 2) + 12 * rows
    gbs = nbytes / (s_ms * 1e-3) / 1e9
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    line = {
        "metric": "decode forward (split-K) GB/s of algorithmic HBM traffic", "value": gbs,
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": s_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "B1 H16 NQ=1 NK=131072 d128 non-causal shared K (decode); step "
                               "= split-K forward + merge",
                   "splits": splits, "bytes_per_step": nbytes,
                   "l2": "keys (537 MB) larger than the 126 MB L2; no flush"},
        "unsplit_ms": u_ms, "speedup_vs_unsplit": u_ms / s_ms,
        "roofline": {"bound": "hbm", "kernel": "streamkl_fwd_keys_kernel (split, keys as MMA rows) + merge",
                     "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": None, "peak_source": "%s hbm_gbs" % peak_src,
                     "note": "achieved = algorithmic bytes per step / CUDA-event time of the step"},
        "clocks": clk,
        "gpu_launches": 2 * args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_chunk(args):
    """Backward (both settings) on the chunk workload (512 query rows per head against 65536
    keys): 64 query tiles for 148 SMs, so the library splits every tile's keys into ranges.
    Reports TFLOP/s of the backward against the measured tensor peak."""
    import torch

    from attention_kl_divergence_02_b200 import binding, inputs

    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--chunk measures one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    binding.load()
    w = inputs.WORKLOADS["chunk"]
    t = inputs.make(w, device=dev)
    B, Hq, NQ, NK, d = w.B, w.Hq, w.NQ, w.NK, w.d
    stream = torch.cuda.current_stream()
    kl, l1, l2 = binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, stream=stream)
    ws_bytes = binding.streamkl_bwd_workspace_bytes(B, Hq, w.Hkv, NQ, NK, d)
    dk_part = B * w.Hkv * ((NK + 127) // 128 * 128) * d * 4
    ws = torch.empty(ws_bytes // 4, dtype=torch.float32, device=dev)
    g = (torch.empty_like(t["q1"]), torch.empty_like(t["k1"]))

    def bwd(mode):
        binding.bwd(mode, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], scale=w.scale,
                    out=g, workspace=ws, stream=stream)

    wa, wb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(args.warmup):
        if i == args.warmup - 1:
            wa.record(stream)
        bwd(1)
        bwd(2)
    wb.record(stream)
    torch.cuda.synchronize()
    warm_ms = wa.elapsed_time(wb)
    st = binding.streamkl_device_status()
    if st != binding.OK:
        raise RuntimeError("device status after warm-up: %s" % binding.status_string(st))

    def timed(mode):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(args.steps):
            bwd(mode)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    probe = ClockProbe(binding, dev)
    torch.cuda.synchronize()
    probe.start(warm_ms * args.steps)
    r0 = torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    m1 = timed(1)
    m2 = timed(2)
    r1 = torch.cuda.Event(enable_timing=True)
    r1.record(stream)
    clk = clocks.stop()
    eff = probe.stop(r0.elapsed_time(r1))
    if eff:
        clk.update(eff)
    st = binding.streamkl_device_status()
    if st != binding.OK:
        raise RuntimeError("device status after the timed region: %s" % binding.status_string(st))
    flops = w.bwd_flops()
    t1, t2 = flops / (m1 * 1e-3) / 1e12, flops / (m2 * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak, peak_label, peak_reason = choose_peak(peaks, peak_src, (m1 + m2) * args.steps * 1e-3, clk)
    line = {
        "metric": "backward TFLOP/s, query chunk against a long context (key-range backward)",
        "value": 2 * flops / ((m1 + m2) * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": m1 + m2,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "B1 H16 NQ=512 NK=65536 d128 non-causal shared K (chunk); step = "
                               "backward P1-fixed + backward P2-fixed",
                   "key_ranges_in_use": ws_bytes > dk_part,
                   "l2": "inputs and dK workspace (0.54 GB) larger than the 126 MB L2; no flush"},
        "bwd_mode1_ms": m1, "bwd_mode1_tflops": t1, "bwd_mode2_ms": m2, "bwd_mode2_tflops": t2,
        "roofline": {"bound": "tensor", "kernel": "bwd_mode1", "achieved": t1, "peak": peak,
                     "unit": "TFLOP/s", "frac": t1 / peak, "traffic": None,
                     "bwd_mode2_frac": t2 / peak, "frac_of_burst": t1 / burst,
                     "peak_source": peak_label, "peak_rule": peak_reason,
                     "note": "achieved = algorithmic FLOPs (8d per pair) / CUDA-event time of the "
                             "call (memset, kernel, dK and dQ converts)"},
        "clocks": clk,
        "gpu_launches": 3 * 2 * args.steps + (1 if eff else 0),
    }
    print(json.dumps(line), flush=True)
    return 0


CONFIG_RUNS = {
    # name: (workload, causal override or None)
    "b2h8n4k": ("b2h8n4k", True),
    "b2h8n4k_noncausal": ("b2h8n4k", False),
    "long64k": ("long64k", None),
    "gqa": ("gqa", None),
    "headline": ("headline", None),
}


def run_config(args):
    """One JSON line for one workload: forward and both backward settings, ms and TFLOP/s per
    call, % of the bf16 peak, the forward's exponential-unit fraction and the fp64 oracle
    timed on a sample of the same workload beside them.  Not the driver's step line: the
    per-workload breakdown behind it."""
    import torch

    from attention_kl_divergence_02_b200 import binding, inputs

    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--config measures one GPU")
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    binding.load()
    wname, causal = CONFIG_RUNS[args.config]
    w = inputs.WORKLOADS[wname]
    if causal is not None:
        w = inputs.variant(w, causal=causal)
    t = inputs.make(w, device=dev)
    B, Hq, NQ, d = w.B, w.Hq, w.NQ, w.d
    stream = torch.cuda.current_stream()
    kl, l1, l2 = (torch.empty((B, Hq, NQ), device=dev) for _ in range(3))
    g = (torch.empty_like(t["q1"]), torch.empty_like(t["k1"]))
    ws = torch.empty(max(16, binding.streamkl_bwd_workspace_bytes(B, Hq, w.Hkv, NQ, w.NK, d)) // 4,
                     device=dev)

    def fwd():
        binding.fwd(t["q1"], t["k1"], t["q2"], t["k2"], scale=w.scale, causal=w.causal,
                    out=(kl, l1, l2), stream=stream)

    def bwd(mode):
        binding.bwd(mode, t["q1"], t["k1"], t["q2"], t["k2"], kl, l1, l2, t["dkl"], scale=w.scale,
                    causal=w.causal, out=g, workspace=ws, stream=stream)

    wa, wb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(args.warmup):
        if i == args.warmup - 1:
            wa.record(stream)
        fwd(); bwd(1); bwd(2)
    wb.record(stream)
    torch.cuda.synchronize()
    warm_step_ms = wa.elapsed_time(wb)
    st = binding.streamkl_device_status()
    if st != binding.OK:
        raise RuntimeError("device status after warm-up: %s" % binding.status_string(st))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    probe = ClockProbe(binding, dev)
    torch.cuda.synchronize()
    probe.start(warm_step_ms * args.steps)
    for k in range(args.steps):
        ev[k][0].record(stream)
        fwd()
        ev[k][1].record(stream)
        bwd(1)
        ev[k][2].record(stream)
        bwd(2)
        ev[k][3].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    eff = probe.stop(ev[0][0].elapsed_time(ev[-1][3]))
    if eff:
        clk.update(eff)
    st = binding.streamkl_device_status()
    if st != binding.OK:
        raise RuntimeError("device status after the timed region: %s" % binding.status_string(st))
    ms = [sum(e[i].elapsed_time(e[i + 1]) for e in ev) / args.steps for i in range(3)]
    total_s = sum(ms) * args.steps * 1e-3
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak, peak_label, peak_reason = choose_peak(peaks, peak_src, total_s, clk)
    fl = [w.fwd_flops(), w.bwd_flops(), w.bwd_flops()]
    tf = [f / (m * 1e-3) / 1e12 for f, m in zip(fl, ms)]
    exp_roof = None
    if not args.skip_exp:
        rates = measure_exp_rates(binding, stream, local)
        exp_roof = exp_roofline(w, ms[0], rates, clk.get("sm_mhz_effective") or clk.get("sm_mhz")
                                or rates["mufu_ex2"]["sm_mhz"])
    line = {
        "metric": "per-workload fwd/bwd ms and TFLOP/s; % of B200 dense bf16 peak",
        "value": sum(fl) / (sum(ms) * 1e-3) / 1e12, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sum(ms),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "%s: %s%s" % (wname, w.note,
                                             "" if causal is None else (" [causal]" if causal else " [non-causal]")),
                   "B": B, "Hq": Hq, "Hkv": w.Hkv, "NQ": NQ, "NK": w.NK, "d": d,
                   "causal": w.causal, "shared_k": w.shared_k},
        "fwd_ms": ms[0], "fwd_tflops": tf[0],
        "bwd_mode1_ms": ms[1], "bwd_mode1_tflops": tf[1],
        "bwd_mode2_ms": ms[2], "bwd_mode2_tflops": tf[2],
        "pct_of_burst_peak": {"fwd": 100 * tf[0] / burst, "bwd_mode1": 100 * tf[1] / burst,
                              "bwd_mode2": 100 * tf[2] / burst,
                              "basis": "%s bf16 %.1f TFLOP/s (burst)" % (peak_src, burst)},
        "roofline": {"bound": "tensor", "peak": peak, "unit": "TFLOP/s", "peak_source": peak_label,
                     "peak_rule": peak_reason, "fwd_frac": tf[0] / peak,
                     "bwd_mode1_frac": tf[1] / peak, "bwd_mode2_frac": tf[2] / peak},
        "exp_roofline": exp_roof,
        "clocks": clk,
        "gpu_launches": 5 * args.steps + (1 if eff else 0),
    }
    if not args.skip_cpu:
        line["cpu_baseline"] = cpu_baseline(w, target_s=10.0)
    print(json.dumps(line), flush=True)
    return 0


def load_traffic(kernel):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary
    (profiles/dram_traffic.txt, lines "<call> <bytes>"), or None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        with open(p) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 2 and not line.startswith("#") and parts[0] == kernel:
                    return int(parts[1])
    except (OSError, ValueError):
        return None
    return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-cpu", action="store_true", help="omit the CPU-oracle baseline leg")
    ap.add_argument("--skip-e2e", action="store_true", help="omit the host-buffer leg")
    ap.add_argument("--skip-exp", action="store_true",
                    help="omit the exponential-throughput probe (and the forward's exp roofline)")
    ap.add_argument("--decode", action="store_true",
                    help="measure the split-K forward on the decode workload instead of the step")
    ap.add_argument("--chunk", action="store_true",
                    help="measure the key-range backward on the chunk workload instead of the step")
    ap.add_argument("--config", choices=sorted(CONFIG_RUNS),
                    help="measure one workload (forward + both backward settings) instead of the step")
    ap.add_argument("--heads", type=int, default=32,
                    help="query/KV heads (32 = the headline workload; fewer only for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.decode:
        return run_decode(args)
    if args.chunk:
        return run_chunk(args)
    if args.config:
        return run_config(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
